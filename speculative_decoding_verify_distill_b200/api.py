"""Python binding of ``libsvd.so`` -- argument marshalling only.

Every entry point has the name of its C function in ``include/svd.h`` and calls it through
ctypes with device pointers taken from torch tensors and the current CUDA stream.  PyTorch is
used for device memory and streams only; all arithmetic runs in the CUDA kernels.  There is no
fallback: if the library is missing or no GPU is present the call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsvd.so")

SVD_OK = 0
STATUS_NAMES = {0: "SVD_OK", 1: "SVD_ERR_INVALID_ARG", 2: "SVD_ERR_ALIGNMENT",
                3: "SVD_ERR_WORKSPACE", 4: "SVD_ERR_CUDA", 5: "SVD_ERR_TIMEOUT",
                6: "SVD_ERR_UNSUPPORTED", 7: "SVD_ERR_TOKEN_RANGE"}
GREEDY, STOCHASTIC = 0, 1
BK_CEIL, BK_FLOOR = 0, 1

# field order of svd_row_info (8 x 4 bytes)
ROW_INFO_FIELDS = ("draft_token", "target_argmax", "accepted", "sample_token", "ratio",
                   "lse_draft", "lse_target", "loss")

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_U64 = ctypes.c_uint64
_SZ = ctypes.c_size_t


class SvdError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__("%s: %s" % (where, STATUS_NAMES.get(code, "status %d" % code)))
        self.code = code


class VerifyDistillArgs(ctypes.Structure):
    """Mirror of ``svd_verify_distill_args``."""
    _fields_ = [
        ("h", _P), ("W1", _P), ("b1", _P), ("w2", _P), ("b2", _F), ("H", _I), ("M", _I),
        ("gamma", _F), ("rnd", _I), ("bk_in", _P),
        ("D", _P), ("T", _P), ("draft_tok", _P), ("B", _I), ("k", _I), ("kt", _I), ("V", _I),
        ("mode", _I), ("temperature", _F), ("seed", _U64), ("step", _U64),
        ("lambda_", _F), ("clip_c", _F), ("grad_scale", _F), ("dlogits_fp32", _I),
        ("bhat", _P), ("bk", _P), ("accept_len", _P), ("emitted", _P), ("n_emitted", _P),
        ("loss_rows", _P), ("loss_total", _P), ("dlogits", _P), ("row_info", _P),
        ("full_k", _I), ("label_proxy", _P), ("label_full", _P), ("head_preact", _P),
    ]


class HeadUpdateArgs(ctypes.Structure):
    """Mirror of ``svd_head_update_args``."""
    _fields_ = [
        ("h", _P), ("label", _P), ("B", _I), ("H", _I), ("M", _I),
        ("W1m", _P), ("b1", _P), ("w2m", _P), ("b2", _P), ("W1", _P), ("w2", _P),
        ("mW1", _P), ("vW1", _P), ("mb1", _P), ("vb1", _P), ("mw2", _P), ("vw2", _P),
        ("mb2", _P), ("vb2", _P), ("step", _I),
        ("lr", _F), ("beta1", _F), ("beta2", _F), ("eps", _F), ("weight_decay", _F),
        ("loss", _P), ("bhat", _P), ("preact", _P),
    ]


class VsArgs(ctypes.Structure):
    """Mirror of ``svd_vs_args`` (include/svd_vocab.h)."""
    _fields_ = [
        ("D", _P), ("T", _P), ("draft_tok", _P), ("bk", _P), ("B", _I), ("k", _I), ("kt", _I),
        ("V", _I), ("v0", _I), ("Vl", _I), ("P", _I), ("rank", _I), ("mode", _I),
        ("temperature", _F), ("seed", _U64), ("step", _U64), ("distill", _I),
        ("lambda_", _F), ("clip_c", _F), ("grad_scale", _F), ("dlogits", _P), ("dlogits_fp32", _I),
        ("loss_rows", _P), ("loss_total", _P), ("accept_len", _P), ("emitted", _P),
        ("n_emitted", _P), ("row_info", _P),
    ]


_lib = None


def lib():
    """The loaded ``libsvd.so`` with argument types declared (raises if absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libsvd.so is not built (%s); run "
                           "`python -m speculative_decoding_verify_distill_b200.build`" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    L.svd_workspace_bytes.argtypes = [_I, _I, _I, _I]
    L.svd_workspace_bytes.restype = _SZ
    L.svd_workspace_reset.argtypes = [_P, _SZ, _P]
    L.svd_length_head.argtypes = [_P, _P, _P, _P, _F, _I, _I, _I, _I, _F, _I, _P, _P, _P, _SZ, _P]
    L.svd_verify.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _U64, _U64, _P, _P, _P, _P,
                             _P, _SZ, _P]
    L.svd_distill_loss_grad.argtypes = [_P, _P, _P, _I, _I, _I, _I, _F, _F, _F, _F, _P, _P, _P, _I,
                                        _P, _SZ, _P]
    L.svd_verify_distill.argtypes = [ctypes.POINTER(VerifyDistillArgs), _P, _SZ, _P]
    L.svd_get_device_error.argtypes = [_P, _P]
    L.svd_status_string.argtypes = [_I]
    L.svd_status_string.restype = ctypes.c_char_p
    L.svd_selftest_wait_timeout.argtypes = [_P, _SZ, _U64, _P]
    L.svd_verify_distill_noalloc.argtypes = [ctypes.POINTER(VerifyDistillArgs), _P, _P]
    L.svd_speedup_report.argtypes = [_P, _P, _P, _I, _I, ctypes.c_double, _P, _P]
    L.svd_length_head_update.argtypes = [ctypes.POINTER(HeadUpdateArgs), _P, _SZ, _P]
    L.svd_vs_exchange_bytes.argtypes = [_I, _I, _I]
    L.svd_vs_exchange_bytes.restype = _SZ
    L.svd_vs_workspace_bytes.argtypes = [_I, _I, _I]
    L.svd_vs_workspace_bytes.restype = _SZ
    L.svd_vs_stats.argtypes = [ctypes.POINTER(VsArgs), _P, _P, _SZ, _P]
    L.svd_vs_resolve.argtypes = [ctypes.POINTER(VsArgs), _P, _P, _P, _SZ, _P]
    L.svd_vs_finish.argtypes = [ctypes.POINTER(VsArgs), _P, _P, _SZ, _P]
    for fn in ("svd_workspace_reset", "svd_length_head", "svd_verify", "svd_distill_loss_grad",
               "svd_verify_distill", "svd_get_device_error", "svd_selftest_wait_timeout",
               "svd_verify_distill_noalloc", "svd_speedup_report", "svd_length_head_update",
               "svd_vs_stats", "svd_vs_resolve", "svd_vs_finish"):
        getattr(L, fn).restype = _I
    _lib = L
    return L


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(code: int, where: str):
    if code != SVD_OK:
        raise SvdError(code, where)


def _bits(t: torch.Tensor) -> torch.Tensor:
    if t.dtype != torch.bfloat16:
        raise TypeError("expected bf16 logits / weights, got %s" % t.dtype)
    return t


class Workspace:
    """Caller-owned scratch for the kernels: zeroed once, reused across calls on one stream."""

    def __init__(self, B: int, k: int, kt: Optional[int] = None, M: int = 0, device=None):
        kt = k if kt is None else kt
        n = int(lib().svd_workspace_bytes(B, k, kt, M))
        self.nbytes = max(n, 256)
        # torch's caching allocator returns 512-byte aligned blocks
        self.buf = torch.zeros(self.nbytes, dtype=torch.uint8, device=device or "cuda")
        assert self.buf.data_ptr() % 256 == 0
        self.shape = (B, k, kt, M)

    def fits(self, B, k, kt, M=0) -> bool:
        return int(lib().svd_workspace_bytes(B, k, kt, M)) <= self.nbytes

    @property
    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())


def _ws(ws, B, k, kt, M, device):
    if ws is None or not ws.fits(B, k, kt, M):
        ws = Workspace(B, k, kt, M, device=device)
    return ws


def svd_workspace_bytes(B: int, k: int, kt: int, M: int = 0) -> int:
    return int(lib().svd_workspace_bytes(B, k, kt, M))


def svd_get_device_error(ws: Workspace, stream=None) -> int:
    return int(lib().svd_get_device_error(ws.ptr, _stream(stream)))


def svd_status_string(code: int) -> str:
    return lib().svd_status_string(int(code)).decode()


def svd_length_head(h, W1, b1, w2, b2: float, k: int, gamma: float = 1.0, rnd: int = BK_CEIL,
                    ws: Optional[Workspace] = None, stream=None):
    """a1: returns (bhat [B] fp32, b_k [B] int32) on h's device."""
    B, H = h.shape
    M = W1.shape[0]
    dev = h.device
    ws = _ws(ws, B, k, k, M, dev)
    bhat = torch.empty(B, dtype=torch.float32, device=dev)
    bk = torch.empty(B, dtype=torch.int32, device=dev)
    _check(lib().svd_length_head(_ptr(_bits(h)), _ptr(_bits(W1)), _ptr(b1), _ptr(_bits(w2)),
                                 float(b2), B, H, M, k, float(gamma), int(rnd), _ptr(bhat),
                                 _ptr(bk), ws.ptr, ws.nbytes, _stream(stream)), "svd_length_head")
    return bhat, bk


def _row_info_tensor(B, kt, dev):
    return torch.empty((B, kt, 8), dtype=torch.int32, device=dev)


def row_info_dict(ri: torch.Tensor) -> dict:
    """Split a [B, kt, 8] int32 row-info buffer into named fields (ints / floats)."""
    out = {}
    for j, name in enumerate(ROW_INFO_FIELDS):
        col = ri[..., j]
        out[name] = col if j < 4 else col.view(torch.float32)
    return out


def svd_verify(D, T, draft_tok, bk, mode: int = GREEDY, temperature: float = 1.0, seed: int = 0,
               step: int = 0, row_info: bool = False, ws: Optional[Workspace] = None, stream=None):
    """a2-a4: truncated verification.  Returns dict(accept_len, emitted, n_emitted[, row_info])."""
    B, k, V = D.shape
    kt = T.shape[1]
    dev = D.device
    ws = _ws(ws, B, k, kt, 0, dev)
    acc = torch.empty(B, dtype=torch.int32, device=dev)
    emitted = torch.empty((B, k + 1), dtype=torch.int32, device=dev)
    ne = torch.empty(B, dtype=torch.int32, device=dev)
    ri = _row_info_tensor(B, kt, dev) if row_info else None
    _check(lib().svd_verify(_ptr(_bits(D)), _ptr(_bits(T)), _ptr(draft_tok), _ptr(bk), B, k, kt, V,
                            int(mode), float(temperature), int(seed), int(step), _ptr(acc),
                            _ptr(emitted), _ptr(ne), _ptr(ri), ws.ptr, ws.nbytes, _stream(stream)),
           "svd_verify")
    out = dict(accept_len=acc, emitted=emitted, n_emitted=ne)
    if ri is not None:
        out["row_info"] = ri
    return out


def svd_distill_loss_grad(D, T, bk, lam: float, clip_c: float, temperature: float = 1.0,
                          grad_scale: float = 1.0, dlogits_fp32: bool = False,
                          ws: Optional[Workspace] = None, stream=None, dlogits=None):
    """a5: returns dict(loss_rows [B,k], loss_total [1], dlogits [B,k,V])."""
    B, k, V = D.shape
    kt = T.shape[1]
    dev = D.device
    ws = _ws(ws, B, k, kt, 0, dev)
    loss_rows = torch.empty((B, k), dtype=torch.float32, device=dev)
    loss_total = torch.empty(1, dtype=torch.float32, device=dev)
    if dlogits is None:
        dlogits = torch.empty((B, k, V), dtype=torch.float32 if dlogits_fp32 else torch.bfloat16,
                              device=dev)
    _check(lib().svd_distill_loss_grad(_ptr(_bits(D)), _ptr(_bits(T)), _ptr(bk), B, k, kt, V,
                                       float(lam), float(clip_c), float(temperature),
                                       float(grad_scale), _ptr(loss_rows), _ptr(loss_total),
                                       _ptr(dlogits), int(bool(dlogits_fp32)), ws.ptr, ws.nbytes,
                                       _stream(stream)), "svd_distill_loss_grad")
    return dict(loss_rows=loss_rows, loss_total=loss_total, dlogits=dlogits)


class VerifyDistill:
    """Preallocated outputs + argument block for repeated fused calls (the benchmark path)."""

    def __init__(self, D, T, *, head=None, bk_in=None, draft_tok=None, mode=GREEDY,
                 temperature=1.0, seed=0, step=0, lam=0.5, clip_c=1.0, grad_scale=1.0,
                 gamma=1.0, rnd=BK_CEIL, dlogits_fp32=False, row_info=False, ws=None,
                 full_k=False, labels=False, head_preact=False):
        B, k, V = D.shape
        kt = T.shape[1]
        dev = D.device
        self.D, self.T, self.head, self.draft_tok, self.bk_in = D, T, head, draft_tok, bk_in
        M = head[1].shape[0] if head is not None else 0
        self.ws = _ws(ws, B, k, kt, M, dev)
        self.bhat = torch.empty(B, dtype=torch.float32, device=dev)
        self.bk = torch.empty(B, dtype=torch.int32, device=dev)
        self.accept_len = torch.empty(B, dtype=torch.int32, device=dev)
        self.emitted = torch.empty((B, k + 1), dtype=torch.int32, device=dev)
        self.n_emitted = torch.empty(B, dtype=torch.int32, device=dev)
        self.loss_rows = torch.empty((B, k), dtype=torch.float32, device=dev)
        self.loss_total = torch.empty(1, dtype=torch.float32, device=dev)
        self.dlogits = torch.empty((B, k, V), dtype=torch.float32 if dlogits_fp32 else torch.bfloat16,
                                   device=dev)
        self.row_info = _row_info_tensor(B, kt, dev) if row_info else None
        # length-head labels: a / b_k as truncated verification sees it, and a / k (full-k mode)
        self.label_proxy = torch.empty(B, dtype=torch.float32, device=dev) if labels else None
        self.label_full = torch.empty(B, dtype=torch.float32, device=dev) if labels else None
        # the head's pre-activations, for an online update that reuses this forward
        self.head_preact = (torch.empty((B, M), dtype=torch.float32, device=dev)
                            if head_preact and head is not None else None)
        a = VerifyDistillArgs()
        if head is not None:
            h, W1, b1, w2, b2 = head
            a.h, a.W1, a.b1, a.w2 = _ptr(_bits(h)), _ptr(_bits(W1)), _ptr(b1), _ptr(_bits(w2))
            a.b2, a.H, a.M = float(b2), h.shape[1], W1.shape[0]
        else:
            if bk_in is None:
                raise ValueError("either head or bk_in is required")
            a.bk_in = _ptr(bk_in)
        a.gamma, a.rnd = float(gamma), int(rnd)
        a.D, a.T, a.draft_tok = _ptr(_bits(D)), _ptr(_bits(T)), _ptr(draft_tok)
        a.B, a.k, a.kt, a.V = B, k, kt, V
        a.mode, a.temperature, a.seed, a.step = int(mode), float(temperature), int(seed), int(step)
        a.lambda_, a.clip_c, a.grad_scale = float(lam), float(clip_c), float(grad_scale)
        a.dlogits_fp32 = int(bool(dlogits_fp32))
        a.bhat, a.bk = _ptr(self.bhat), _ptr(self.bk)
        a.accept_len, a.emitted, a.n_emitted = _ptr(self.accept_len), _ptr(self.emitted), _ptr(self.n_emitted)
        a.loss_rows, a.loss_total, a.dlogits = _ptr(self.loss_rows), _ptr(self.loss_total), _ptr(self.dlogits)
        a.row_info = _ptr(self.row_info)
        a.full_k = int(bool(full_k))
        a.label_proxy, a.label_full = _ptr(self.label_proxy), _ptr(self.label_full)
        a.head_preact = _ptr(self.head_preact)
        self.args = a

    def set_step(self, step: int):
        self.args.step = int(step)

    def __call__(self, stream=None):
        _check(lib().svd_verify_distill(ctypes.byref(self.args), self.ws.ptr, self.ws.nbytes,
                                        _stream(stream)), "svd_verify_distill")
        return self

    def outputs(self) -> dict:
        out = dict(bhat=self.bhat, bk=self.bk, accept_len=self.accept_len, emitted=self.emitted,
                   n_emitted=self.n_emitted, loss_rows=self.loss_rows, loss_total=self.loss_total,
                   dlogits=self.dlogits)
        if self.row_info is not None:
            out["row_info"] = self.row_info
        if self.label_proxy is not None:
            out["label_proxy"] = self.label_proxy
            out["label_full"] = self.label_full
        if self.head_preact is not None:
            out["head_preact"] = self.head_preact
        return out


def svd_verify_distill(D, T, **kw) -> dict:
    """a1-a5 in one call; keyword arguments as in :class:`VerifyDistill`."""
    return VerifyDistill(D, T, **kw)().outputs()


class LengthHeadTrainer:
    """Online AdamW training of the length head through ``svd_length_head_update``.

    Holds fp32 master weights, AdamW moments and the bf16 copies the forward serves
    (``W1``, ``w2``; pass ``head()`` to :class:`VerifyDistill`).  Defaults: learning rate 2e-4
    (the pages' value), betas (0.9, 0.999), eps 1e-8, weight decay 0.01.
    """

    def __init__(self, W1, b1, w2, b2: float, B: int, lr=2e-4, betas=(0.9, 0.999), eps=1e-8,
                 weight_decay=0.01):
        dev = W1.device
        M, H = W1.shape
        self.B, self.H, self.M = B, H, M
        self.W1m = W1.float().contiguous().clone()
        self.b1 = (torch.zeros(M, device=dev) if b1 is None else b1.float().clone()).contiguous()
        self.w2m = w2.float().contiguous().clone()
        self.b2 = torch.full((1,), float(b2), dtype=torch.float32, device=dev)
        self.W1 = self.W1m.to(torch.bfloat16).contiguous()
        self.w2 = self.w2m.to(torch.bfloat16).contiguous()
        self.moments = [torch.zeros_like(t) for t in (self.W1m, self.W1m, self.b1, self.b1,
                                                      self.w2m, self.w2m, self.b2, self.b2)]
        self.loss = torch.zeros(1, dtype=torch.float32, device=dev)
        self.bhat = torch.zeros(B, dtype=torch.float32, device=dev)
        self.ws = Workspace(B, 1, 1, M, device=dev)
        self.step_count = 0
        self.hyper = (float(lr), float(betas[0]), float(betas[1]), float(eps), float(weight_decay))

    def head(self, h):
        """The (h, W1, b1, w2, b2) tuple for :class:`VerifyDistill` (b2 read back from device)."""
        return (h, self.W1, self.b1, self.w2, float(self.b2.item()))

    def step(self, h, label, stream=None, preact=None, bhat=None):
        """One AdamW step on l = mean_b (bhat_b - label_b)^2; returns (loss, bhat) tensors.

        With ``preact`` and ``bhat`` (the ``head_preact`` and ``bhat`` of a
        :class:`VerifyDistill` step on the same h with this trainer's current weights), the
        step reuses that forward instead of running its own."""
        if h.shape != (self.B, self.H):
            raise ValueError("h must be [B, H] = [%d, %d]" % (self.B, self.H))
        if (preact is None) != (bhat is None):
            raise ValueError("preact and bhat go together")
        self.step_count += 1
        a = HeadUpdateArgs()
        bhat_buf = self.bhat
        if preact is not None:
            if preact.shape != (self.B, self.M) or preact.dtype != torch.float32:
                raise ValueError("preact must be fp32 [B, M]")
            if bhat.shape != (self.B,) or bhat.dtype != torch.float32 or not bhat.is_contiguous():
                raise ValueError("bhat must be a contiguous fp32 [B] tensor")
            bhat_buf = bhat            # read by the update, not written
            a.preact = _ptr(preact.contiguous())
        lab = label.float().contiguous()
        self._label = lab   # alive until the launch is enqueued
        a.h, a.label = _ptr(_bits(h)), _ptr(lab)
        a.B, a.H, a.M = self.B, self.H, self.M
        a.W1m, a.b1, a.w2m, a.b2 = _ptr(self.W1m), _ptr(self.b1), _ptr(self.w2m), _ptr(self.b2)
        a.W1, a.w2 = _ptr(self.W1), _ptr(self.w2)
        (a.mW1, a.vW1, a.mb1, a.vb1, a.mw2, a.vw2, a.mb2, a.vb2) = [_ptr(t) for t in self.moments]
        a.step = self.step_count
        a.lr, a.beta1, a.beta2, a.eps, a.weight_decay = self.hyper
        a.loss, a.bhat = _ptr(self.loss), _ptr(bhat_buf)
        _check(lib().svd_length_head_update(ctypes.byref(a), self.ws.ptr, self.ws.nbytes,
                                            _stream(stream)), "svd_length_head_update")
        return self.loss, bhat_buf


REPORT_FIELDS = ("tau_measured", "acc", "tau_model", "eta_model", "eta_measured", "mean_bk",
                 "mean_accept", "B")


def svd_speedup_report(accept_len, bk, n_emitted, k: int, rho: float = 0.0, stream=None):
    """E[tau] (measured and modelled), Acc, eta and per-position acceptance as a fp64 CUDA
    tensor [8 + k]; see :func:`report_dict` for the field names."""
    out = torch.empty(8 + int(k), dtype=torch.float64, device=accept_len.device)
    _check(lib().svd_speedup_report(_ptr(accept_len), _ptr(bk), _ptr(n_emitted),
                                    int(accept_len.numel()), int(k), float(rho), _ptr(out),
                                    _stream(stream)), "svd_speedup_report")
    return out


def report_dict(out) -> dict:
    v = out.double().cpu().tolist()
    d = dict(zip(REPORT_FIELDS, v[:8]))
    d["alpha"] = v[8:]
    return d


NOALLOC_SCRATCH_BYTES = 4 << 20


def svd_verify_distill_noalloc(vd: VerifyDistill, status_out=None, stream=None) -> None:
    """The fused call on the library's static per-device scratch instead of ``vd.ws``.

    For callers that cannot allocate device memory on their path (a runtime that has claimed
    nearly all HBM for its own pools, or a host program without a device allocator): the C
    entry point allocates nothing.  ``status_out`` is an optional one-element int32/uint32 CUDA
    tensor that receives the device status word.  Overlapping calls on one device race on the
    shared scratch; the first call per device must come before any stream capture.
    """
    _check(lib().svd_verify_distill_noalloc(ctypes.byref(vd.args), _ptr(status_out),
                                            _stream(stream)), "svd_verify_distill_noalloc")


def svd_selftest_wait_timeout(ws: Workspace, limit_ns: int, stream=None) -> None:
    _check(lib().svd_selftest_wait_timeout(ws.ptr, ws.nbytes, int(limit_ns), _stream(stream)),
           "svd_selftest_wait_timeout")


INF = math.inf


# ------------------------------------------------------------------------------------------
# vocab-sharded pass (include/svd_vocab.h)
# ------------------------------------------------------------------------------------------
def svd_vs_exchange_bytes(B: int, kt: int, which: int) -> int:
    return int(lib().svd_vs_exchange_bytes(B, kt, which))


def svd_vs_workspace_bytes(B: int, k: int, kt: int) -> int:
    return int(lib().svd_vs_workspace_bytes(B, k, kt))


class VocabShard:
    """One rank's part of the vocab-sharded verify-and-distill pass.

    ``D`` [B, k, Vl] and ``T`` [B, kt, Vl] are this rank's slices (ids ``v0 .. v0+Vl-1``) of
    the logit rows.  The three calls ``svd_vs_stats``, ``svd_vs_resolve`` and ``svd_vs_finish``
    read and write the exchange buffers ``send1``/``recv1`` and ``send2``/``recv2`` (uint8,
    rank r's records at block r of ``recv*``); moving ``send*`` of every rank into ``recv*``
    is the caller's all-gather (``vocab_parallel``)."""

    def __init__(self, D, T, bk, *, V: int, v0: int, P: int, rank: int, draft_tok=None,
                 mode: int = GREEDY, temperature: float = 1.0, seed: int = 0, step: int = 0,
                 distill: bool = True, lam: float = 0.5, clip_c: float = 1.0,
                 grad_scale: float = 1.0, dlogits_fp32: bool = False, row_info: bool = False):
        B, k, Vl = D.shape
        kt = T.shape[1]
        dev = D.device
        self.shape = (B, k, kt, V, v0, Vl, P, rank)
        self.mode = int(mode)
        self.distill = bool(distill)
        self._keep = [_bits(D), _bits(T), bk, draft_tok]
        i32 = dict(dtype=torch.int32, device=dev)
        self.accept_len = torch.empty(B, **i32)
        self.emitted = torch.empty((B, k + 1), **i32)
        self.n_emitted = torch.empty(B, **i32)
        self.loss_rows = torch.empty((B, k), dtype=torch.float32, device=dev) if distill else None
        self.loss_total = torch.empty(1, dtype=torch.float32, device=dev) if distill else None
        self.dlogits = (torch.empty((B, k, Vl), dtype=torch.float32 if dlogits_fp32 else torch.bfloat16,
                                    device=dev) if distill else None)
        self.row_info = _row_info_tensor(B, kt, dev) if row_info else None
        u8 = dict(dtype=torch.uint8, device=dev)
        n1, n2 = svd_vs_exchange_bytes(B, kt, 1), svd_vs_exchange_bytes(B, kt, 2)
        self.send1 = torch.empty(max(n1, 16), **u8)
        self.recv1 = torch.empty(max(P * n1, 16), **u8)
        self.send2 = torch.empty(max(n2, 16), **u8)
        self.recv2 = torch.empty(max(P * n2, 16), **u8)
        nw = max(svd_vs_workspace_bytes(B, k, kt), 256)
        self.ws = torch.zeros(nw, **u8)
        assert self.ws.data_ptr() % 256 == 0
        a = VsArgs()
        a.D, a.T = _ptr(D), _ptr(T)
        a.draft_tok, a.bk = _ptr(draft_tok), _ptr(bk)
        a.B, a.k, a.kt, a.V, a.v0, a.Vl, a.P, a.rank = B, k, kt, V, v0, Vl, P, rank
        a.mode, a.temperature, a.seed, a.step = int(mode), float(temperature), int(seed), int(step)
        a.distill = 1 if distill else 0
        a.lambda_, a.clip_c, a.grad_scale = float(lam), float(clip_c), float(grad_scale)
        a.dlogits, a.dlogits_fp32 = _ptr(self.dlogits), 1 if dlogits_fp32 else 0
        a.loss_rows, a.loss_total = _ptr(self.loss_rows), _ptr(self.loss_total)
        a.accept_len, a.emitted, a.n_emitted = _ptr(self.accept_len), _ptr(self.emitted), _ptr(self.n_emitted)
        a.row_info = _ptr(self.row_info)
        self.args = a

    @property
    def stochastic(self) -> bool:
        return self.mode == STOCHASTIC

    def set_step(self, step: int):
        self.args.step = int(step)

    def _ws(self):
        return ctypes.c_void_p(self.ws.data_ptr()), self.ws.numel()

    def stats(self, stream=None):
        w, n = self._ws()
        _check(lib().svd_vs_stats(ctypes.byref(self.args), _ptr(self.send1), w, n, _stream(stream)),
               "svd_vs_stats")

    def resolve(self, stream=None):
        w, n = self._ws()
        _check(lib().svd_vs_resolve(ctypes.byref(self.args), _ptr(self.recv1), _ptr(self.send2), w, n,
                                    _stream(stream)), "svd_vs_resolve")

    def finish(self, stream=None):
        w, n = self._ws()
        _check(lib().svd_vs_finish(ctypes.byref(self.args), _ptr(self.recv2), w, n, _stream(stream)),
               "svd_vs_finish")

    def device_error(self, stream=None) -> int:
        return int(lib().svd_get_device_error(ctypes.c_void_p(self.ws.data_ptr()), _stream(stream)))

    def outputs(self) -> dict:
        out = dict(accept_len=self.accept_len, emitted=self.emitted, n_emitted=self.n_emitted)
        if self.distill:
            out.update(loss_rows=self.loss_rows, loss_total=self.loss_total, dlogits=self.dlogits)
        if self.row_info is not None:
            out["row_info"] = self.row_info
        return out
