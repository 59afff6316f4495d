"""svd_verify_distill_noalloc: the fused call on the library's static per-device scratch.

The entry point serves callers that cannot allocate device memory on their path (a runtime
that has claimed nearly all HBM for its own pools, a host program without a device allocator).
Its results must equal those of svd_verify_distill with a caller workspace, call after call,
since both run the same kernels.  This file is named so that pytest collects it last: the
first call on a device does the scratch set-up, and it must work both in a fresh process and
after every other test has used the library.
"""
import ctypes

import numpy as np
import pytest
import torch

from speculative_decoding_verify_distill_b200 import api
from speculative_decoding_verify_distill_b200 import build as svd_build
from speculative_decoding_verify_distill_b200 import synthetic as syn
from tests import parity as P


@pytest.fixture(scope="module")
def L():
    svd_build.build()
    return api.lib()


def test_rejections_before_any_launch(L):
    """Argument and size errors return before the scratch is set up (no CUDA call is made):
    every argument check runs first, then the size check."""
    assert L.svd_verify_distill_noalloc(None, None, None) == 1
    fake = ctypes.c_void_p(0x1000)   # never dereferenced
    a = api.VerifyDistillArgs()
    a.bk_in = a.D = a.T = a.bk = a.accept_len = a.emitted = a.n_emitted = fake
    a.loss_total = a.dlogits = fake
    a.k, a.kt, a.V, a.temperature, a.lambda_, a.clip_c, a.grad_scale = 16, 16, 1024, 1.0, 0.5, 1.0, 1.0
    # a workspace beyond the static scratch: 20000 x 16 row records alone take 10 MB
    a.B = 20000
    assert api.svd_workspace_bytes(a.B, a.k, a.kt, 0) > api.NOALLOC_SCRATCH_BYTES
    assert L.svd_verify_distill_noalloc(ctypes.byref(a), None, None) == 3
    # a shape the fused call rejects keeps its argument error; an empty batch is a no-op
    a.B, a.k = 0, 0
    assert L.svd_verify_distill_noalloc(ctypes.byref(a), None, None) == 1
    a.k = 16
    assert L.svd_verify_distill_noalloc(ctypes.byref(a), None, None) == 0   # empty batch
    # bad arguments on a shape too large for the scratch: the argument error wins, because
    # every argument is checked before the size, the scratch or the stream is touched
    a.B = 20000
    for field, bad in (("mode", 7), ("temperature", float("nan")), ("k", 33), ("kt", 18),
                       ("lambda_", 1.5), ("clip_c", -1.0), ("full_k", 2)):
        good = getattr(a, field)
        setattr(a, field, bad)
        assert L.svd_verify_distill_noalloc(ctypes.byref(a), None, None) == 1, field
        setattr(a, field, good)
    assert L.svd_verify_distill_noalloc(ctypes.byref(a), None, None) == 3


def _snapshot(vd):
    return {k: v.clone() for k, v in vd.outputs().items()}


def _assert_same(got, want, what):
    for name in ("bk", "accept_len", "emitted", "n_emitted"):
        assert torch.equal(got[name], want[name]), (what, name)
    for name in ("bhat", "loss_rows", "loss_total"):
        P.assert_close(got[name].cpu().numpy(), want[name].cpu().numpy(), "%s %s" % (what, name))
    P.assert_close(got["dlogits"].float().cpu().numpy(), want["dlogits"].float().cpu().numpy(),
                   "%s dlogits" % what)
    g, r = got["row_info"].cpu(), want["row_info"].cpu()
    assert torch.equal(g[..., :4], r[..., :4]), what


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("case", ["tiny_greedy", "qwen_stochastic_b24"])
def test_noalloc_matches_workspace_call_twice(L, case):
    if case == "tiny_greedy":
        w = syn.WORKLOADS["tiny"]
    else:
        w = syn.WORKLOADS["stochastic_qwen_b64"].with_(B=24, kt=17)
    D, T = syn.make_logits(w)
    h, W1, b1, w2, b2 = syn.make_head(w)
    dev = "cuda"
    head = (h.to(dev), W1.to(dev), b1.to(dev), w2.to(dev), b2)
    draft = syn.sample_draft_tokens(D, w.tau, 5).to(dev) if w.mode == 1 else None
    Dd, Td = D.to(dev), T.to(dev)
    kw = dict(head=head, draft_tok=draft, mode=w.mode, temperature=w.tau, seed=w.philox_seed,
              lam=w.lam, clip_c=w.clip_c, row_info=True)
    ref = api.VerifyDistill(Dd, Td, **kw)
    na = api.VerifyDistill(Dd, Td, **kw)
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)

    # two calls in a row on the static scratch, then the workspace call for each step
    na.set_step(0)
    api.svd_verify_distill_noalloc(na, status_out=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    first = _snapshot(na)
    na.set_step(1)
    status.fill_(-1)
    api.svd_verify_distill_noalloc(na, status_out=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    second = _snapshot(na)

    for step, got in ((0, first), (1, second)):
        ref.set_step(step)
        ref()
        torch.cuda.synchronize()
        assert api.svd_get_device_error(ref.ws) == 0
        _assert_same(got, _snapshot(ref), "%s step %d" % (case, step))
    if w.mode == 1:
        # different Philox steps give different stochastic decisions somewhere in the batch
        assert not (torch.equal(first["emitted"], second["emitted"])
                    and torch.equal(first["row_info"][..., 3], second["row_info"][..., 3]))


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_noalloc_reports_device_error_and_recovers(L):
    """A draft token outside [0, V) is reported through status_out; the next call starts clean."""
    w = syn.WORKLOADS["tiny"].with_(mode=1)
    D, T = syn.make_logits(w)
    dev = "cuda"
    bk = torch.full((w.B,), w.k, dtype=torch.int32, device=dev)
    good = syn.sample_draft_tokens(D, w.tau, 9).to(dev)
    bad = good.clone()
    bad[1, 2] = w.V + 5
    Dd, Td = D.to(dev), T.to(dev)
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    vd_bad = api.VerifyDistill(Dd, Td, bk_in=bk, draft_tok=bad, mode=1)
    api.svd_verify_distill_noalloc(vd_bad, status_out=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 7   # SVD_ERR_TOKEN_RANGE
    vd_good = api.VerifyDistill(Dd, Td, bk_in=bk, draft_tok=good, mode=1)
    api.svd_verify_distill_noalloc(vd_good, status_out=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = api.VerifyDistill(Dd, Td, bk_in=bk, draft_tok=good, mode=1)()
    torch.cuda.synchronize()
    for name in ("accept_len", "emitted", "n_emitted"):
        assert torch.equal(vd_good.outputs()[name], ref.outputs()[name]), name
    P.assert_close(vd_good.loss_total.cpu().numpy(), ref.loss_total.cpu().numpy(), "loss_total")
