"""CPU oracle for the AdaFlash verify-and-distill path (fp64, plain loops).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package.  The product library never links, loads or calls
it, and it shares no code with the CUDA path.  The arithmetic lives in ``svd_oracle.c``; this
module only compiles that file with gcc and marshals numpy arrays through ctypes.

Which pins hold each function (see ``tests/test_oracle_*.py``):
  * ``length_head``  -- torch fp64 Linear/ReLU/sigmoid; hand-computed ceil/floor edges.
  * ``row_stats``    -- scipy logsumexp, numpy argmax (first index), brute force at V = 8.
  * ``verify``       -- draft == target gives full acceptance; hand-built mismatches; exact
                        emission law P(emit = v) = p_v at V = 8 (chi-square); the closed form
                        E[tau] = (1 - A^(k+1)) / (1 - A) of the Pith review's referee report.
  * ``distill``      -- KL = 0 when draft == target; RKL >= 0; K_c <= RKL; c = inf equals torch
                        kl_div; lambda = 1 equals torch cross_entropy; a hand-derived V = 2
                        golden case; finite differences; torch autograd; sum of gradient = 0.
  * ``length_head_update`` -- torch fp64 autograd of an independent expression of the loss;
                        a hand-derived one-unit case; three AdamW steps against torch.optim.AdamW.
  * ``speedup_report`` -- hand-counted small cases; all-accepted and all-rejected limits; the
                        closed form recovered from geometric accept lengths (i.i.d. rate A).
  * ``philox``       -- bit-exact agreement with cuRAND's Philox4x32-10: its host generator
                        (CPU suite: both key words, counter words 0-2) and its device API
                        (GPU suite: counter words 2-3 from 64-bit subsequences); uniformity,
                        independence and avalanche tests.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "svd_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``svd_oracle.c`` into ``liboracle.so`` (gcc, IEEE fp64, OpenMP over sequences)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
               "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    i32, u64, f64 = ctypes.c_int, ctypes.c_uint64, ctypes.c_double
    lib.orc_set_threads.argtypes = [i32]
    lib.orc_max_threads.restype = i32
    lib.orc_philox4x32_10.argtypes = [P, P, P]
    lib.orc_philox_words.argtypes = [u64, u64, i32, i32, P]
    lib.orc_length_head.argtypes = [P, P, P, P, f64, i32, i32, i32, i32, f64, i32, P, P, P]
    lib.orc_length_head.restype = i32
    lib.orc_row_stats.argtypes = [P, i32, f64, P, P, P]
    lib.orc_speedup_report.argtypes = [P, P, P, i32, i32, f64, P]
    lib.orc_length_head_update.argtypes = [P, P, i32, i32, i32, P, P, P, f64, P, P, P, P,
                                           P, P, P, P, P, P, P, P, i32, f64, f64, f64, f64, f64,
                                           P, P, P, P, P, P]
    lib.orc_length_head_update.restype = i32
    lib.orc_speedup_report.restype = i32
    lib.orc_verify.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, f64, u64, u64,
                               P, P, P, P, P, P, P, P, P]
    lib.orc_verify.restype = i32
    lib.orc_distill.argtypes = [P, P, P, i32, i32, i32, i32, f64, f64, f64, f64,
                                P, P, P, P, P, P]
    lib.orc_distill.restype = i32
    lib.orc_distill_f64.argtypes = lib.orc_distill.argtypes
    lib.orc_distill_f64.restype = i32
    lib.orc_row_stats_f64.argtypes = [P, i32, f64, P, P, P]
    lib.orc_clip_band.argtypes = [P, P, P, i32, i32, i32, i32, f64, f64, f64, P, P, P, P]
    lib.orc_clip_band.restype = i32
    lib.orc_sample_inverse_cdf.argtypes = [P, i32, f64, P]
    lib.orc_sample_inverse_cdf.restype = ctypes.c_int32
    lib.orc_expected_tokens.argtypes = [f64, i32]
    lib.orc_expected_tokens.restype = f64
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _bits(x) -> np.ndarray:
    """bf16 data as a C-contiguous uint16 array (accepts torch bf16 tensors or uint16 arrays)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16
            return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(x)
    assert a.dtype == np.uint16
    return a


def set_threads(n: int) -> None:
    _load().orc_set_threads(int(n))


def max_threads() -> int:
    return int(_load().orc_max_threads())


def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32))
    kk = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    out = np.zeros(4, dtype=np.uint32)
    _load().orc_philox4x32_10(_ptr(c), _ptr(kk), _ptr(out))
    return out


def philox_words(seed: int, step: int, seq: int, pos: int) -> np.ndarray:
    out = np.zeros(4, dtype=np.uint32)
    _load().orc_philox_words(seed, step, seq, pos, _ptr(out))
    return out


def length_head(h, W1, b1, w2, b2: float, k: int, gamma: float = 1.0, rnd: int = 0):
    """Returns (bhat [B] f64, b_k [B] int32, z [B] f64)."""
    hb, Wb, wb = _bits(h), _bits(W1), _bits(w2)
    B, H = hb.shape
    M = Wb.shape[0]
    b1a = None if b1 is None else np.ascontiguousarray(np.asarray(b1, dtype=np.float64))
    bhat = np.zeros(B, np.float64)
    bk = np.zeros(B, np.int32)
    z = np.zeros(B, np.float64)
    rc = _load().orc_length_head(_ptr(hb), _ptr(Wb), _ptr(b1a), _ptr(wb), float(b2), B, H, M, k,
                                 float(gamma), int(rnd), _ptr(bhat), _ptr(bk), _ptr(z))
    if rc != 0:
        raise ValueError("oracle length_head: bad arguments")
    return bhat, bk, z


def row_stats(x, tau: float = 1.0):
    """(max, argmax, lse) of one row, given as bf16 (torch bf16 / uint16 bits) or float64."""
    if isinstance(x, np.ndarray) and x.dtype == np.float64:
        xb, fn = np.ascontiguousarray(x.reshape(-1)), _load().orc_row_stats_f64
    else:
        xb, fn = _bits(x).reshape(-1), _load().orc_row_stats
    mx = np.zeros(1, np.float64)
    am = np.zeros(1, np.int32)
    lse = np.zeros(1, np.float64)
    fn(_ptr(xb), xb.size, float(tau), _ptr(mx), _ptr(am), _ptr(lse))
    return float(mx[0]), int(am[0]), float(lse[0])


def sample_inverse_cdf(w, u: float):
    """(token, margin) of the ascending-id inverse-CDF sampler on weights w (float64)."""
    wa = np.ascontiguousarray(np.asarray(w, dtype=np.float64))
    margin = np.zeros(1, np.float64)
    tok = _load().orc_sample_inverse_cdf(_ptr(wa), wa.size, float(u), _ptr(margin))
    return int(tok), float(margin[0])


def verify(D, T, draft, bk, mode: int, tau: float = 1.0, seed: int = 0, step: int = 0,
           seq_ids=None):
    """Truncated verification.  D [B,k,V], T [B,kt,V] bf16; bk [B]; draft [B,k] or None;
    seq_ids [B] = index of each sequence in its full batch (Philox counter), default 0..B-1.

    Returns a dict of numpy arrays: accept_len, emitted, n_emitted and the per-row diagnostics
    row_x, row_y, row_ratio, row_u, row_acc, fix_margin.
    """
    Db, Tb = _bits(D), _bits(T)
    B, k, V = Db.shape
    kt = Tb.shape[1]
    assert Tb.shape[0] == B and Tb.shape[2] == V
    bka = np.ascontiguousarray(np.asarray(bk, dtype=np.int32))
    dr = None if draft is None else np.ascontiguousarray(np.asarray(draft, dtype=np.int32))
    sid = None if seq_ids is None else np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int32))
    out = dict(
        accept_len=np.zeros(B, np.int32), emitted=np.zeros((B, k + 1), np.int32),
        n_emitted=np.zeros(B, np.int32), row_x=np.zeros((B, k), np.int32),
        row_y=np.zeros((B, kt), np.int32), row_ratio=np.zeros((B, k), np.float64),
        row_u=np.zeros((B, k), np.float64), row_acc=np.zeros((B, k), np.int32),
        fix_margin=np.zeros(B, np.float64))
    rc = _load().orc_verify(_ptr(Db), _ptr(Tb), _ptr(dr), _ptr(bka), _ptr(sid), B, k, kt, V, int(mode),
                            float(tau), int(seed), int(step), _ptr(out["accept_len"]),
                            _ptr(out["emitted"]), _ptr(out["n_emitted"]), _ptr(out["row_x"]),
                            _ptr(out["row_y"]), _ptr(out["row_ratio"]), _ptr(out["row_u"]),
                            _ptr(out["row_acc"]), _ptr(out["fix_margin"]))
    if rc == 1:
        raise ValueError("oracle verify: bad arguments")
    out["token_error"] = rc == 2
    return out


def distill(D, T, bk, lam: float, clip_c: float, tau: float = 1.0, grad_scale: float = 1.0,
            want_grad: bool = True):
    """OPD loss and gradient.  D [B,k,V], T [B,kt,V] as bf16 (torch bf16 or uint16 bits) or as
    float64 numpy arrays.  Returns dict: loss_rows [B,k], loss_total, dlogits [B,k,V] f64 (or
    None), rkl_rows, kc_rows, ce_rows."""
    f64_inputs = isinstance(D, np.ndarray) and D.dtype == np.float64
    if f64_inputs:
        Db = np.ascontiguousarray(D)
        Tb = np.ascontiguousarray(np.asarray(T, dtype=np.float64))
        fn = _load().orc_distill_f64
    else:
        Db, Tb = _bits(D), _bits(T)
        fn = _load().orc_distill
    B, k, V = Db.shape
    kt = Tb.shape[1]
    bka = np.ascontiguousarray(np.asarray(bk, dtype=np.int32))
    loss_rows = np.zeros((B, k), np.float64)
    tot = np.zeros(1, np.float64)
    g = np.zeros((B, k, V), np.float64) if want_grad else None
    rkl = np.zeros((B, k), np.float64)
    kc = np.zeros((B, k), np.float64)
    ce = np.zeros((B, k), np.float64)
    rc = fn(_ptr(Db), _ptr(Tb), _ptr(bka), B, k, kt, V, float(lam),
                             float(clip_c), float(tau), float(grad_scale), _ptr(loss_rows),
                             _ptr(tot), _ptr(g), _ptr(rkl), _ptr(kc), _ptr(ce))
    if rc != 0:
        raise ValueError("oracle distill: bad arguments")
    return dict(loss_rows=loss_rows, loss_total=float(tot[0]), dlogits=g, rkl_rows=rkl,
                kc_rows=kc, ce_rows=ce)


def clip_band(D, T, bk, clip_c: float, tau: float = 1.0, band_rel: float = 1e-5,
              want_mask: bool = True):
    """Entries whose clip decision d_v <= c is within fp32 error of flipping (see
    ``orc_clip_band``).  D [B,k,V], T [B,kt,V] bf16; returns dict n_band [B,k] int32,
    dS [B,k] and dK [B,k] (bounds of the effect of flipped decisions on S and on K_c), and
    band [B,k,V] bool (or None)."""
    Db, Tb = _bits(D), _bits(T)
    B, k, V = Db.shape
    kt = Tb.shape[1]
    bka = np.ascontiguousarray(np.asarray(bk, dtype=np.int32))
    n = np.zeros((B, k), np.int32)
    dS = np.zeros((B, k), np.float64)
    dK = np.zeros((B, k), np.float64)
    m = np.zeros((B, k, V), np.uint8) if want_mask else None
    rc = _load().orc_clip_band(_ptr(Db), _ptr(Tb), _ptr(bka), B, k, kt, V, float(clip_c),
                               float(tau), float(band_rel), _ptr(n), _ptr(dS), _ptr(dK), _ptr(m))
    if rc != 0:
        raise ValueError("oracle clip_band: bad arguments")
    return dict(n_band=n, dS=dS, dK=dK, band=None if m is None else m.astype(bool))


def expected_tokens(A: float, k: int) -> float:
    return float(_load().orc_expected_tokens(float(A), int(k)))


def length_head_update(h, label, W1, b1, w2, b2: float, state: dict, step: int,
                       lr: float = 2e-4, beta1: float = 0.9, beta2: float = 0.999,
                       eps: float = 1e-8, wd: float = 0.01) -> dict:
    """One AdamW step of the length head on l = mean_b (bhat_b - label_b)^2.

    h, W1, w2: bf16 (the served forward weights); b1: fp32/fp64 [M]; b2: float.  ``state``
    holds fp64 numpy arrays W1m, b1m, w2m, b2m (masters) and mW1, vW1, mb1, vb1, mw2, vw2,
    mb2, vb2 (AdamW moments); they are updated in place.  Returns loss, bhat and the gradients.
    """
    hb, Wb, wb = _bits(h), _bits(W1), _bits(w2)
    B, H = hb.shape
    M = Wb.shape[0]
    lab = np.ascontiguousarray(np.asarray(label, np.float64))
    b1a = np.ascontiguousarray(np.asarray(b1, np.float64))
    for key in ("W1m", "b1m", "w2m", "b2m", "mW1", "vW1", "mb1", "vb1", "mw2", "vw2", "mb2", "vb2"):
        arr = state[key]
        assert arr.dtype == np.float64 and arr.flags["C_CONTIGUOUS"], key
    loss = np.zeros(1, np.float64)
    bhat = np.zeros(B, np.float64)
    gW1 = np.zeros((M, H), np.float64)
    gb1 = np.zeros(M, np.float64)
    gw2 = np.zeros(M, np.float64)
    gb2 = np.zeros(1, np.float64)
    S = state
    rc = _load().orc_length_head_update(
        _ptr(hb), _ptr(lab), B, H, M, _ptr(Wb), _ptr(b1a), _ptr(wb), float(b2),
        _ptr(S["W1m"]), _ptr(S["b1m"]), _ptr(S["w2m"]), _ptr(S["b2m"]),
        _ptr(S["mW1"]), _ptr(S["vW1"]), _ptr(S["mb1"]), _ptr(S["vb1"]),
        _ptr(S["mw2"]), _ptr(S["vw2"]), _ptr(S["mb2"]), _ptr(S["vb2"]),
        int(step), float(lr), float(beta1), float(beta2), float(eps), float(wd),
        _ptr(loss), _ptr(bhat), _ptr(gW1), _ptr(gb1), _ptr(gw2), _ptr(gb2))
    if rc != 0:
        raise ValueError("oracle length_head_update: bad arguments")
    return dict(loss=float(loss[0]), bhat=bhat, gW1=gW1, gb1=gb1, gw2=gw2, gb2=float(gb2[0]))


def speedup_report(accept_len, bk, n_emitted, k: int, rho: float) -> np.ndarray:
    """fp64 [8 + k]: measured E[tau], Acc, model E[tau], eta (model), eta (measured), mean b_k,
    mean accepted length, B, then the per-position acceptance rates (see svd_oracle.c)."""
    lib = _load()
    a = np.ascontiguousarray(accept_len, np.int32)
    n = np.ascontiguousarray(bk, np.int32)
    e = np.ascontiguousarray(n_emitted, np.int32)
    out = np.zeros(8 + int(k), np.float64)
    rc = lib.orc_speedup_report(a.ctypes.data, n.ctypes.data, e.ctypes.data, len(a), int(k),
                                float(rho), out.ctypes.data)
    if rc != 0:
        raise ValueError("orc_speedup_report: bad arguments")
    return out
