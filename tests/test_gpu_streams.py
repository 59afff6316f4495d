"""Calls on several CUDA streams at once, each with its own workspace (the C ABI says such calls
are reentrant): every output must equal, bit for bit, the same call made alone.  The fused
pass is deterministic (every sum in a fixed order), so nothing but interference could change a
bit.  Also a length-head update on a third stream while two fused calls run."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from speculative_decoding_verify_distill_b200 import api
from speculative_decoding_verify_distill_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def _case(seed: int, B: int, k: int, V: int):
    g = torch.Generator(device="cuda").manual_seed(seed)
    T = (2.0 * torch.randn((B, k, V), generator=g, device="cuda")).to(torch.bfloat16)
    D = (T.float() + 0.8 * torch.randn((B, k, V), generator=g, device="cuda")).to(torch.bfloat16)
    return D, T


def _snapshot(vd: api.VerifyDistill) -> dict:
    return {name: t.clone() for name, t in vd.outputs().items() if t is not None}


def _same(a: dict, b: dict):
    assert a.keys() == b.keys()
    for name in a:
        assert torch.equal(a[name], b[name]), name


@pytest.mark.parametrize("mode", [api.GREEDY, api.STOCHASTIC])
def test_fused_calls_on_two_streams(mode):
    w = syn.WORKLOADS["greedy_qwen_b32"]
    h, W1, b1, w2, b2 = (t.cuda() if torch.is_tensor(t) else t for t in syn.make_head(w))
    calls = []
    for seed, V in ((1, 151936), (2, 128256)):
        D, T = _case(seed, w.B, w.k, V)
        draft = None
        if mode == api.STOCHASTIC:
            # any draft tokens serve (the test compares a call with itself): Gumbel-max on the GPU
            gum = torch.empty(D.shape, dtype=torch.float32, device="cuda").exponential_(
                generator=torch.Generator(device="cuda").manual_seed(seed + 10)).log().neg()
            draft = torch.argmax(D.float() + gum, dim=-1).to(torch.int32)
            del gum
        calls.append(api.VerifyDistill(D, T, head=(h, W1, b1, w2, b2), draft_tok=draft, mode=mode,
                                       seed=seed, lam=0.5, clip_c=1.0))
    # alone, one after the other
    alone = []
    for vd in calls:
        vd()
        torch.cuda.synchronize()
        assert api.svd_get_device_error(vd.ws) == 0
        alone.append(_snapshot(vd))
    # together: each on its own stream, several rounds enqueued before any synchronization
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    torch.cuda.synchronize()
    for _ in range(4):
        for vd, s in zip(calls, streams):
            vd(s)
    torch.cuda.synchronize()
    for vd, ref in zip(calls, alone):
        assert api.svd_get_device_error(vd.ws) == 0
        _same(_snapshot(vd), ref)


def test_head_update_alongside_fused_calls():
    w = syn.WORKLOADS["greedy_qwen_b32"]
    h, W1, b1, w2, b2 = syn.make_head(w)
    hd = h.cuda()
    D, T = _case(3, w.B, w.k, w.V)
    head = (hd, W1.cuda(), b1.cuda(), w2.cuda(), b2)
    vd = api.VerifyDistill(D, T, head=head, lam=0.5, clip_c=1.0)
    label = torch.rand(w.B, generator=torch.Generator().manual_seed(4)).cuda()
    # the update alone, from a fresh copy of the weights
    tr_alone = api.LengthHeadTrainer(W1.cuda(), b1.cuda(), w2.cuda(), b2, w.B)
    tr_alone.step(hd, label)
    vd()
    torch.cuda.synchronize()
    ref_vd = _snapshot(vd)
    ref_w = [t.clone() for t in (tr_alone.W1m, tr_alone.w2m, tr_alone.b1, tr_alone.W1, tr_alone.w2)]
    # the same update on its own stream while the fused call runs twice on another
    tr = api.LengthHeadTrainer(W1.cuda(), b1.cuda(), w2.cuda(), b2, w.B)
    s_rows, s_upd = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    vd(s_rows)
    with torch.cuda.stream(s_upd):
        tr.step(hd, label, stream=s_upd)
    vd(s_rows)
    torch.cuda.synchronize()
    assert api.svd_get_device_error(vd.ws) == 0
    _same(_snapshot(vd), ref_vd)
    for got, want in zip((tr.W1m, tr.w2m, tr.b1, tr.W1, tr.w2), ref_w):
        assert torch.equal(got, want)
    assert np.isfinite(tr.loss.item())
