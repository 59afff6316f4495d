"""svd_length_head_update (one AdamW step of the length head on mean_b (bhat_b - a*_b)^2)
against the fp64 oracle, step by step: before every step the oracle starts from the GPU's
state (fp32 masters, moments and the served bf16 copies), so each step is compared alone."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verify_distill_b200 import api
from speculative_decoding_verify_distill_b200 import synthetic as syn

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

LR = 2e-4


@pytest.fixture(scope="module", autouse=True)
def _built():
    from speculative_decoding_verify_distill_b200 import build
    build.build()
    oracle.build()


def _np(t):
    return t.detach().double().cpu().numpy().copy()


def _oracle_state(tr):
    names = ("mW1", "vW1", "mb1", "vb1", "mw2", "vw2", "mb2", "vb2")
    st = dict(W1m=_np(tr.W1m), b1m=_np(tr.b1), w2m=_np(tr.w2m), b2m=_np(tr.b2))
    st.update({n: _np(t) for n, t in zip(names, tr.moments)})
    return st


def _check_step(tr, h, label, step):
    st = _oracle_state(tr)
    W1f, w2f = tr.W1.cpu(), tr.w2.cpu()
    ref = oracle.length_head_update(h.cpu(), label.cpu().double().numpy(), W1f, st["b1m"].copy(),
                                    w2f, float(st["b2m"][0]), st, step, lr=LR)
    loss, bhat = tr.step(h, label)
    torch.cuda.synchronize()
    assert loss.item() == pytest.approx(ref["loss"], rel=2e-5)
    np.testing.assert_allclose(bhat.cpu().numpy(), ref["bhat"], rtol=2e-5, atol=1e-6)
    # parameters: exact up to the gradient's fp32 rounding; entries whose gradient is at the
    # rounding noise (|g| < 1e-4 of the largest) may take Adam's sign-like step either way
    for name, gpu, gname in (("W1m", tr.W1m, "gW1"), ("b1m", tr.b1, "gb1"), ("w2m", tr.w2m, "gw2")):
        got, want = _np(gpu), st[name]
        g = np.abs(ref[gname])
        ambiguous = g < 1e-4 * g.max()
        bad = (np.abs(got - want) > 1e-3 * LR + 1e-6 * np.abs(want)) & ~ambiguous
        assert not bad.any(), (name, step, int(bad.sum()), np.argwhere(bad)[:3])
        # ambiguous entries still move by at most Adam's largest step (lr * 3 within three steps)
        assert (np.abs(got - want)[ambiguous] <= 3.0 * LR + 1e-6 * np.abs(want)[ambiguous]).all()
        # a sanity bound: near-zero gradients are a small minority (dead or barely live units)
        assert ambiguous.mean() < 0.02, (name, ambiguous.mean())
    assert _np(tr.b2)[0] == pytest.approx(st["b2m"][0], abs=1e-3 * LR)
    # moments
    np.testing.assert_allclose(_np(tr.moments[0]), st["mW1"], rtol=1e-3, atol=1e-9)
    np.testing.assert_allclose(_np(tr.moments[1]), st["vW1"], rtol=2e-3, atol=1e-14)
    # the served copies are the RNE bf16 of the fp32 masters, bit for bit
    assert torch.equal(tr.W1, tr.W1m.to(torch.bfloat16))
    assert torch.equal(tr.w2, tr.w2m.to(torch.bfloat16))
    return ref


@pytest.mark.parametrize("B,H,M", [(32, 512, 64), (7, 300, 37), (128, 4096, 256), (200, 1024, 128),
                                   (300, 520, 70)])
def test_update_steps_match_oracle(B, H, M):
    """Three AdamW steps against the oracle.  B = 200 and 300 take the backward through more than
    one 128-sequence chunk (the later chunks staged after the first); H = 520 and M = 70 leave
    partial 64-column and 64-unit blocks (plain loads where a staged row would run past H or M)."""
    w = syn.WORKLOADS["ragged_qwen_b128"].with_(B=B, H=H, M=M)
    h, W1, b1, w2, b2 = syn.make_head(w)
    tr = api.LengthHeadTrainer(W1.cuda(), b1.cuda(), w2.cuda(), b2, B, lr=LR)
    g = torch.Generator().manual_seed(B + H + M)
    label = torch.rand(B, generator=g, dtype=torch.float32).cuda()
    hd = h.cuda()
    for step in (1, 2, 3):
        _check_step(tr, hd, label, step)


def test_update_on_labels_from_a_verification_step():
    w = syn.WORKLOADS["greedy_qwen_b32"]
    D, T = syn.make_logits(w)
    h, W1, b1, w2, b2 = syn.make_head(w)
    tr = api.LengthHeadTrainer(W1.cuda(), b1.cuda(), w2.cuda(), b2, w.B, lr=LR)
    hd = h.cuda()
    vd = api.VerifyDistill(D.cuda(), T.cuda(), head=tr.head(hd), lam=w.lam, clip_c=w.clip_c,
                           full_k=True, labels=True)
    vd()
    torch.cuda.synchronize()
    for label in (vd.label_proxy.clone(), vd.label_full.clone()):
        _check_step(tr, hd, label, tr.step_count + 1)


def test_bad_arguments():
    a = api.HeadUpdateArgs()
    L = api.lib()
    import ctypes
    assert L.svd_length_head_update(None, None, 0, None) == 1
    assert L.svd_length_head_update(ctypes.byref(a), None, 0, None) == 1   # B = 0, null pointers


def test_update_reusing_the_verification_forward():
    """The fused call's head pre-activations and bhat stand in for the update's own forward:
    the step then matches the oracle's (which recomputes the forward) as closely as a step
    with its own forward does."""
    w = syn.WORKLOADS["greedy_qwen_b32"]
    D, T = syn.make_logits(w)
    h, W1, b1, w2, b2 = syn.make_head(w)
    tr = api.LengthHeadTrainer(W1.cuda(), b1.cuda(), w2.cuda(), b2, w.B, lr=LR)
    hd = h.cuda()
    for step in (1, 2):
        vd = api.VerifyDistill(D.cuda(), T.cuda(), head=tr.head(hd), lam=w.lam, clip_c=w.clip_c,
                               labels=True, head_preact=True)
        vd()
        torch.cuda.synchronize()
        label = vd.label_proxy.clone()
        st = _oracle_state(tr)
        ref = oracle.length_head_update(h, label.cpu().double().numpy(), tr.W1.cpu(),
                                        st["b1m"].copy(), tr.w2.cpu(), float(st["b2m"][0]), st,
                                        tr.step_count + 1, lr=LR)
        loss, bhat = tr.step(hd, label, preact=vd.head_preact, bhat=vd.bhat)
        torch.cuda.synchronize()
        assert loss.item() == pytest.approx(ref["loss"], rel=2e-5)
        np.testing.assert_allclose(bhat.cpu().numpy(), ref["bhat"], rtol=2e-5, atol=1e-6)
        for name, gpu, gname in (("W1m", tr.W1m, "gW1"), ("b1m", tr.b1, "gb1"), ("w2m", tr.w2m, "gw2")):
            got, want = _np(gpu), st[name]
            g = np.abs(ref[gname])
            ambiguous = g < 1e-4 * g.max()
            bad = (np.abs(got - want) > 1e-3 * LR + 1e-6 * np.abs(want)) & ~ambiguous
            assert not bad.any(), (name, step, int(bad.sum()))
        np.testing.assert_allclose(_np(tr.moments[0]), st["mW1"], rtol=1e-3, atol=1e-9)
        assert torch.equal(tr.W1, tr.W1m.to(torch.bfloat16))
