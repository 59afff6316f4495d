"""GPU parity on edge cases: ragged and unaligned vocabularies, extreme k / b_k, argmax ties
across cluster ranks, temperatures, clipping extremes, the three single-purpose entry points,
determinism, workspace reuse and the device-side error paths (none of which faults a GPU)."""
import math

import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verify_distill_b200 import api
from speculative_decoding_verify_distill_b200 import synthetic as syn
from tests import parity as P
from tests.test_gpu_parity import compare_sequences, cuda, ri_fields

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from speculative_decoding_verify_distill_b200 import build
    build.build()
    oracle.build()


def make_case(B, k, kt, V, seed, sigma=0.8):
    g = torch.Generator().manual_seed(seed)
    T = 2.0 * torch.randn((B, kt, V), generator=g)
    D = T[:, :k] + sigma * torch.randn((B, k, V), generator=g)
    return D.to(torch.bfloat16), T.to(torch.bfloat16)


def fused(D, T, bk, *, draft=None, mode=0, tau=1.0, lam=0.5, clip_c=1.0, seed=5, step=0,
          dl_fp32=False, grad_scale=1.0):
    vd = api.VerifyDistill(cuda(D), cuda(T), bk_in=cuda(bk), draft_tok=None if draft is None else cuda(draft),
                           mode=mode, temperature=tau, seed=seed, step=step, lam=lam, clip_c=clip_c,
                           grad_scale=grad_scale, dlogits_fp32=dl_fp32, row_info=True)
    vd()
    torch.cuda.synchronize()
    assert api.svd_get_device_error(vd.ws) == 0
    return vd


def full_compare(vd, D, T, bk, *, draft=None, mode=0, tau=1.0, lam=0.5, clip_c=1.0, seed=5,
                 step=0, dl_fp32=False, grad_scale=1.0):
    out = vd.outputs()
    seqs = list(range(D.shape[0]))
    st = compare_sequences(out, D, T, draft, np.asarray(bk), seqs, mode=mode, tau=tau, seed=seed,
                           step=step, lam=lam, clip_c=clip_c, grad_scale=grad_scale,
                           grad_seqs=seqs, dl_fp32=dl_fp32)
    r = oracle.distill(D, T, np.asarray(bk), lam, clip_c, tau, grad_scale, want_grad=False)
    P.assert_close(out["loss_total"].cpu().numpy()[0], r["loss_total"], "loss_total")
    return st


@pytest.mark.parametrize("V", [1, 7, 8, 9, 1000, 1024, 1031, 4104, 16384, 16392, 40960, 100000,
                               200003, 262144, 262152, 327680])
def test_vocab_sizes_greedy(V):
    B, k = 3, 4
    D, T = make_case(B, k, k, V, seed=V)
    bk = torch.tensor([1, 3, 4], dtype=torch.int32)
    vd = fused(D, T, bk)
    full_compare(vd, D, T, bk)


@pytest.mark.parametrize("V", [7, 1000, 1024, 40960])
def test_vocab_sizes_stochastic(V):
    B, k = 64, 3
    D, T = make_case(B, k, k + 1, V, seed=V + 1, sigma=1.5)
    draft = syn.sample_draft_tokens_batched(D, 1.0, V)
    bk = syn.random_bk(B, k, V)
    vd = fused(D, T, bk, draft=draft, mode=1, seed=42, step=7)
    full_compare(vd, D, T, bk, draft=draft, mode=1, seed=42, step=7)


@pytest.mark.parametrize("k,kt", [(1, 1), (1, 2), (32, 32), (32, 33), (5, 6)])
def test_block_sizes(k, kt):
    B, V = 4, 2048
    D, T = make_case(B, k, kt, V, seed=k * 100 + kt)
    for bk in (torch.full((B,), 1, dtype=torch.int32), torch.full((B,), k, dtype=torch.int32),
               syn.random_bk(B, k, k + kt)):
        vd = fused(D, T, bk)
        full_compare(vd, D, T, bk)
    # draft == target on every verified row: everything accepted (kt = k: no bonus at b_k = k)
    D2 = T[:, :k].contiguous()
    bkf = torch.full((B,), k, dtype=torch.int32)
    vd = fused(D2, T, bkf)
    acc = vd.accept_len.cpu().numpy()
    assert (acc == k).all()
    assert (vd.n_emitted.cpu().numpy() == (k + 1 if kt == k + 1 else k)).all()


@pytest.mark.parametrize("k,kt", [(1, 2), (32, 33), (5, 6)])
def test_block_sizes_stochastic(k, kt):
    # the draw lands on the first rejected row or, with every draft accepted, on the bonus row
    # (row 32 when k = 32: the last emitted slot)
    B, V = 6, 2048
    D, T = make_case(B, k, kt, V, seed=k * 10 + kt, sigma=1.0)
    for bk, DD in ((syn.random_bk(B, k, k + 3), D),
                   (torch.full((B,), k, dtype=torch.int32), T[:, :k].contiguous())):
        draft = syn.sample_draft_tokens_batched(DD, 1.0, k + kt)
        vd = fused(DD, T, bk, draft=draft, mode=1, seed=5, step=2)
        full_compare(vd, DD, T, bk, draft=draft, mode=1, seed=5, step=2)
    assert (vd.accept_len.cpu().numpy() == k).all()        # draft == target: all accepted
    assert (vd.n_emitted.cpu().numpy() == k + 1).all()     # ... and the bonus token drawn
    assert (vd.emitted.cpu().numpy()[:, k] >= 0).all()


@pytest.mark.parametrize("B", [4096, 4097])
@pytest.mark.parametrize("mode", [0, 1])
def test_batch_size_boundary_of_the_compact_lists(B, mode):
    # up to 4096 sequences the row pass keeps b_k and the loaded / zero-row prefixes in shared
    # memory and hands out work dynamically; above, it walks (sequence, row) slots in a fixed order
    k, V = 3, 64
    D, T = make_case(B, k, k + 1, V, seed=B + mode)
    bk = syn.random_bk(B, k, B + 7)
    draft = syn.sample_draft_tokens_batched(D, 1.0, B) if mode == 1 else None
    vd = fused(D, T, bk, draft=draft, mode=mode, seed=11)
    full_compare(vd, D, T, bk, draft=draft, mode=mode, seed=11)
    g = vd.outputs()["dlogits"].cpu()
    for b in range(0, B, 97):   # gradient rows past b_k are zero
        n = int(bk[b])
        if n < k:
            assert int(torch.count_nonzero(g[b, n:])) == 0


def test_argmax_ties_across_cluster_ranks():
    # V = 40960 runs as a cluster of two CTAs: ties are placed in both halves and in one vector
    B, k, V = 1, 4, 40960
    D, T = make_case(B, k, k + 1, V, seed=3)
    Df, Tf = D.float(), T.float()
    top = 40.0  # exactly representable in bf16, above every random value
    for ids, row in (([30000, 5000, 20479, 20480], 0), ([20480, 40959], 1), ([9, 8, 15], 2),
                     ([40959], 3)):
        for x in ids:
            Df[0, row, x] = top
            Tf[0, row, x] = top
    Tf[0, 4, [100, 99]] = top
    D, T = Df.to(torch.bfloat16), Tf.to(torch.bfloat16)
    bk = torch.tensor([4], dtype=torch.int32)
    vd = fused(D, T, bk)
    full_compare(vd, D, T, bk)
    ri = ri_fields(vd.row_info)
    assert list(ri["target_argmax"][0]) == [5000, 20480, 8, 40959, 99]
    assert list(ri["draft_token"][0, :4]) == [5000, 20480, 8, 40959]


@pytest.mark.parametrize("tau", [0.7, 1.5])
def test_temperature(tau):
    D, T = make_case(3, 4, 4, 3000, seed=11)
    bk = torch.tensor([4, 2, 3], dtype=torch.int32)
    vd = fused(D, T, bk, tau=tau, lam=0.8, clip_c=0.01)
    full_compare(vd, D, T, bk, tau=tau, lam=0.8, clip_c=0.01)
    draft = syn.sample_draft_tokens_batched(D, tau, 9)
    vd = fused(D, T, bk, draft=draft, mode=1, tau=tau, lam=0.8, clip_c=0.01, seed=1)
    full_compare(vd, D, T, bk, draft=draft, mode=1, tau=tau, lam=0.8, clip_c=0.01, seed=1)


@pytest.mark.parametrize("clip_c,lam", [(0.0, 0.0), (1e-4, 0.3), (0.01, 0.8), (math.inf, 0.0),
                                        (0.1, 1.0)])
def test_clipping_extremes_fp32_grad(clip_c, lam):
    D, T = make_case(2, 3, 3, 2056, seed=21, sigma=2.0)
    bk = torch.tensor([3, 2], dtype=torch.int32)
    vd = fused(D, T, bk, lam=lam, clip_c=clip_c, dl_fp32=True, grad_scale=0.125)
    st = full_compare(vd, D, T, bk, lam=lam, clip_c=clip_c, dl_fp32=True, grad_scale=0.125)
    # the element-wise comparison covers (almost) every entry of the verified rows, c = 0 included
    print("clip c=%g: %d band entries, %d compared" % (clip_c, st["clip_band"], st["clip_compared"]))
    assert st["clip_compared"] >= 0.99 * (st["clip_compared"] + st["clip_band"])


def test_single_purpose_entry_points():
    B, k, V = 6, 5, 5000
    D, T = make_case(B, k, k + 1, V, seed=31)
    bk = syn.random_bk(B, k, 31)
    # verify only, greedy, draft = argmax
    out = api.svd_verify(cuda(D), cuda(T), None, cuda(bk), api.GREEDY, 1.0, 0, 0, row_info=True)
    torch.cuda.synchronize()
    ref = oracle.verify(D, T, None, bk.numpy(), 0)
    assert np.array_equal(out["accept_len"].cpu().numpy(), ref["accept_len"])
    assert np.array_equal(out["emitted"].cpu().numpy(), ref["emitted"])
    assert np.array_equal(out["n_emitted"].cpu().numpy(), ref["n_emitted"])
    # verify only, greedy, caller tokens
    draft = syn.sample_draft_tokens_batched(D, 1.0, 4)
    out = api.svd_verify(cuda(D), cuda(T), cuda(draft), cuda(bk), api.GREEDY, 1.0, 0, 0)
    ref = oracle.verify(D, T, draft.numpy(), bk.numpy(), 0)
    assert np.array_equal(out["emitted"].cpu().numpy(), ref["emitted"])
    # verify only, stochastic
    out = api.svd_verify(cuda(D), cuda(T), cuda(draft), cuda(bk), api.STOCHASTIC, 1.0, 99, 3,
                         row_info=True)
    ref = oracle.verify(D, T, draft.numpy(), bk.numpy(), 1, 1.0, 99, 3)
    em = out["emitted"].cpu().numpy()
    for b in range(B):
        n = int(bk[b])
        tie = any(abs(ref["row_u"][b, i] - min(1, ref["row_ratio"][b, i])) < P.TIE_U for i in range(n))
        if not tie and not np.array_equal(em[b], ref["emitted"][b]):
            assert ref["fix_margin"][b] < P.TIE_SAMPLE, (b, em[b], ref["emitted"][b])
    # distill only
    for dl32 in (False, True):
        o = api.svd_distill_loss_grad(cuda(D), cuda(T), cuda(bk), 0.5, 0.05, 1.0, 1.0, dl32)
        torch.cuda.synchronize()
        r = oracle.distill(D, T, bk.numpy(), 0.5, 0.05, 1.0)
        P.assert_close(o["loss_rows"].cpu().numpy(), r["loss_rows"], "loss_rows")
        P.assert_close(o["loss_total"].cpu().numpy()[0], r["loss_total"], "loss_total")
        if dl32:
            P.assert_close(o["dlogits"].cpu().numpy(), r["dlogits"], "dlogits")
        else:
            P.assert_bf16_grad(o["dlogits"].cpu(), r["dlogits"], "dlogits")


def test_length_head_ragged_shapes():
    for B, H, M in ((5, 255, 100), (17, 4096, 64), (1, 16, 1), (40, 1000, 300)):
        g = torch.Generator().manual_seed(B * H + M)
        h = (3 * torch.randn((B, H), generator=g)).to(torch.bfloat16)
        W1 = (0.05 * torch.randn((M, H), generator=g)).to(torch.bfloat16)
        w2 = (0.1 * torch.randn((M,), generator=g)).to(torch.bfloat16)
        b1 = 0.01 * torch.randn((M,), generator=g)
        for rnd in (0, 1):
            bhat, bk = api.svd_length_head(cuda(h), cuda(W1), cuda(b1), cuda(w2), 0.05, 16, 1.0, rnd)
            torch.cuda.synchronize()
            rb, rk, _ = oracle.length_head(h, W1, b1.double().numpy(), w2, 0.05, 16, 1.0, rnd)
            near = P.bk_near_integer(rb, 16)
            assert np.array_equal(bk.cpu().numpy()[~near], rk[~near])
            P.assert_close(bhat.cpu().numpy(), rb, "bhat", rtol=1e-4, atol=1e-6)


def test_determinism_and_workspace_reuse():
    w = syn.WORKLOADS["tiny"]
    D, T = syn.make_logits(w)
    h, W1, b1, w2, b2 = syn.make_head(w)
    vd = api.VerifyDistill(cuda(D), cuda(T), head=(cuda(h), cuda(W1), cuda(b1), cuda(w2), b2),
                           lam=0.5, clip_c=1.0, row_info=True)
    first = {k: v.clone() for k, v in vd().outputs().items()}
    for _ in range(3):
        again = vd().outputs()
    torch.cuda.synchronize()
    for k_, v in first.items():
        assert torch.equal(v, again[k_]), k_
    # every ticket back at zero, status word clear
    hdr = vd.ws.buf[:256].view(torch.int32).cpu().numpy()
    assert (hdr[:3] == 0).all()


def test_device_errors_are_reported_not_faulted():
    D, T = make_case(2, 3, 3, 1024, seed=1)
    bk = torch.tensor([3, 2], dtype=torch.int32)
    ws = api.Workspace(2, 3, 3)
    bad = torch.tensor([[1, 2, 1024], [0, -1, 5]], dtype=torch.int32)
    api.svd_verify(cuda(D), cuda(T), cuda(bad), cuda(bk), api.STOCHASTIC, 1.0, 0, 0, ws=ws)
    assert api.svd_get_device_error(ws) == 7
    assert api.svd_get_device_error(ws) == 0         # read clears it
    # a verification length outside [1, k] coming from device memory
    api.svd_workspace_reset = getattr(api, "svd_workspace_reset", None)
    ws2 = api.Workspace(2, 3, 3)
    api.svd_verify(cuda(D), cuda(T), None, cuda(torch.tensor([0, 9], dtype=torch.int32)),
                   api.GREEDY, 1.0, 0, 0, ws=ws2)
    assert api.svd_get_device_error(ws2) == 1
    # bounded wait: gives up after 1 ms and records a timeout; the context stays usable
    ws3 = api.Workspace(1, 1, 1)
    api.svd_selftest_wait_timeout(ws3, 1_000_000)
    assert api.svd_get_device_error(ws3) == 5
    x = torch.ones(4, device="cuda") * 2
    torch.cuda.synchronize()
    assert float(x.sum()) == 8.0


def test_empty_batch():
    D = torch.empty((0, 4, 64), dtype=torch.bfloat16, device="cuda")
    T = torch.empty((0, 4, 64), dtype=torch.bfloat16, device="cuda")
    bk = torch.empty((0,), dtype=torch.int32, device="cuda")
    assert api.lib().svd_verify(None, None, None, None, 0, 4, 4, 64, 0, 1.0, 0, 0, None, None,
                                None, None, None, 0, None) == 0


@pytest.mark.parametrize("B,H,M,V", [(5, 272, 100, 20000), (17, 4096, 64, 16392),
                                     (40, 1000, 300, 40960), (3, 16, 1, 151936),
                                     (40, 8192, 64, 40960), (9, 2048, 96, 8000)])
def test_fused_head_ragged_shapes(B, H, M, V):
    """The length head inside the row pass on partial sequence / unit tiles (B % 16, M % 64 not
    zero), and the separate head kernel before it where H % 16 != 0: b_k, bhat and everything
    downstream against the oracle.  H = 8192 splits wider than one staging chunk of the row pass
    (two chunks per unit), and V = 8000 takes the small-vocabulary shape, whose 8 KB staging area
    holds 32 columns of a unit at a time."""
    k = 6
    g = torch.Generator().manual_seed(B * 7 + H + M)
    h = (3 * torch.randn((B, H), generator=g)).to(torch.bfloat16)
    W1 = (0.05 * torch.randn((M, H), generator=g)).to(torch.bfloat16)
    w2 = (0.1 * torch.randn((M,), generator=g)).to(torch.bfloat16)
    b1 = 0.01 * torch.randn((M,), generator=g)
    D, T = make_case(B, k, k, V, seed=B + M, sigma=0.9)
    vd = api.VerifyDistill(cuda(D), cuda(T), head=(cuda(h), cuda(W1), cuda(b1), cuda(w2), 0.05),
                           lam=0.5, clip_c=0.5, row_info=True, head_preact=True)
    vd()
    torch.cuda.synchronize()
    assert api.svd_get_device_error(vd.ws) == 0
    out = vd.outputs()
    rb, rk, _ = oracle.length_head(h, W1, b1.double().numpy(), w2, 0.05, k, 1.0, 0)
    near = P.bk_near_integer(rb, k)
    bk = out["bk"].cpu().numpy()
    assert np.array_equal(bk[~near], rk[~near])
    P.assert_close(out["bhat"].cpu().numpy(), rb, "bhat", rtol=1e-4, atol=1e-6)
    # the pre-activations W1 h + b1 the head hands to an online update
    pre = (h.double() @ W1.double().T + b1.double()).numpy()
    P.assert_close(out["head_preact"].cpu().numpy(), pre, "head_preact", rtol=1e-4, atol=1e-4)
    full_compare(vd, D, T, bk, lam=0.5, clip_c=0.5)
