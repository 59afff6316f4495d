"""GPU parity of the vocab-sharded pass (include/svd_vocab.h) against the fp64 oracle on whole
rows: splitting the vocabulary over P ranks must not change what a row computes.

The P ranks run on one device (``vocab_parallel.run_emulated``: every rank's three calls in
rank order, device copies in place of the all-gathers).  Besides the oracle comparison, every
rank must hold bit-identical row results (the decisions are taken independently on each rank
from the same gathered records)."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verify_distill_b200 import api
from speculative_decoding_verify_distill_b200 import synthetic as syn
from speculative_decoding_verify_distill_b200 import vocab_parallel as vp
from tests import parity as P
from tests.test_gpu_parity import compare_sequences, ri_fields

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from speculative_decoding_verify_distill_b200 import build
    build.build()
    oracle.build()


def run_sharded(D, T, bk, Pn, *, draft=None, align=8, slices=None, **kw):
    """Shards D [B,k,V] and T [B,kt,V] (host, bf16) over Pn emulated ranks and runs one step.
    Returns the rank-0 outputs with the gradient slices joined along V, and the shards."""
    B, k, V = D.shape
    slices = slices or vp.vocab_slices(V, Pn, align)
    bk_d = bk.to(torch.int32).cuda() if torch.is_tensor(bk) else torch.from_numpy(np.asarray(bk, np.int32)).cuda()
    dr = None if draft is None else (draft if torch.is_tensor(draft) else torch.from_numpy(draft)).to(torch.int32).cuda()
    shards = []
    for r, (v0, n) in enumerate(slices):
        shards.append(api.VocabShard(D[..., v0:v0 + n].contiguous().cuda(),
                                     T[..., v0:v0 + n].contiguous().cuda(), bk_d, V=V, v0=v0,
                                     P=len(slices), rank=r, draft_tok=dr, row_info=True, **kw))
    vp.run_emulated(shards)
    torch.cuda.synchronize()
    for s in shards:
        assert s.device_error() == 0
    ref = shards[0].outputs()
    for s in shards[1:]:
        o = s.outputs()
        for name in ("accept_len", "emitted", "n_emitted", "row_info"):
            assert torch.equal(o[name], ref[name]), name
        if s.distill:
            assert torch.equal(o["loss_rows"], ref["loss_rows"])
            assert torch.equal(o["loss_total"], ref["loss_total"])
    out = dict(ref)
    if shards[0].distill:
        out["dlogits"] = torch.cat([s.dlogits for s in shards], dim=2)
    return out, shards


def rand_case(B, k, kt, V, seed, sigma=0.7, scale=2.0):
    """Seeded bf16 logits: T ~ scale N(0,1) plus a shared log-rank bias, D = T + sigma N(0,1)."""
    g = torch.Generator().manual_seed(seed)
    bias = -torch.log1p(torch.randperm(V, generator=g).to(torch.float32))
    T = scale * torch.randn((B, kt, V), generator=g) + bias
    D = T[:, :k] + sigma * torch.randn((B, k, V), generator=g)
    return D.to(torch.bfloat16), T.to(torch.bfloat16)


# ------------------------------------------------------------------------------------------
# small cases, every sequence element by element
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("Pn,align", [(1, 8), (2, 8), (3, 8), (8, 8), (3, 1), (5, 1)])
def test_tiny_greedy_sharded(Pn, align):
    w = syn.WORKLOADS["tiny"]
    D, T = syn.make_logits(w)
    bk = syn.random_bk(w.B, w.k, 5)
    for dl32 in (False, True):
        out, _ = run_sharded(D, T, bk, Pn, align=align, temperature=w.tau, lam=w.lam,
                             clip_c=w.clip_c, dlogits_fp32=dl32)
        seqs = list(range(w.B))
        compare_sequences(out, D, T, None, bk.numpy(), seqs, mode=0, tau=w.tau, seed=0, step=0,
                          lam=w.lam, clip_c=w.clip_c, grad_seqs=seqs, dl_fp32=dl32)
        r = oracle.distill(D, T, bk.numpy(), w.lam, w.clip_c, w.tau, want_grad=False)
        P.assert_close(out["loss_total"].cpu().numpy()[0], r["loss_total"], "loss_total")


@pytest.mark.parametrize("Pn", [2, 4])
@pytest.mark.parametrize("kt_extra", [0, 1])
def test_small_stochastic_sharded(Pn, kt_extra):
    B, k, V = 24, 6, 2000
    D, T = rand_case(B, k, k + kt_extra, V, 31 + Pn, sigma=0.9)
    draft = syn.sample_draft_tokens(D, 1.0, 11)
    bk = syn.random_bk(B, k, 9)
    out, _ = run_sharded(D, T, bk, Pn, draft=draft, mode=api.STOCHASTIC, seed=77, step=3,
                         lam=0.5, clip_c=1.0)
    compare_sequences(out, D, T, draft, bk.numpy(), list(range(B)), mode=1, tau=1.0, seed=77,
                      step=3, lam=0.5, clip_c=1.0, grad_seqs=[0, 5, 23])
    # after the max-combine: the drawn token on its row (the first rejected row, else the
    # bonus row), equal to the emitted one; no token on any other row
    ri = ri_fields(out["row_info"])
    acc = out["accept_len"].cpu().numpy()
    em = out["emitted"].cpu().numpy()
    for b in range(B):
        a, nb = int(acc[b]), int(bk[b])
        st = ri["sample_token"][b].copy()
        if a < nb or nb < st.shape[0]:
            assert st[a] == em[b, a] and 0 <= st[a] < V, (b, a, st[a], em[b, a])
            st[a] = -1
        assert (st == -1).all(), (b, ri["sample_token"][b])


@pytest.mark.parametrize("clip_c,lam", [(0.02, 0.0), (0.1, 0.5), (float("inf"), 0.0), (0.0, 1.0),
                                        (0.0, 0.0), (1e-4, 0.3)])
def test_clipping_sharded(clip_c, lam):
    # wide noise makes many entries reach the clip bound
    B, k, V = 6, 4, 3000
    D, T = rand_case(B, k, k, V, 5, sigma=3.0)
    bk = torch.tensor([1, 2, 3, 4, 4, 2], dtype=torch.int32)
    out, _ = run_sharded(D, T, bk, 3, lam=lam, clip_c=clip_c, temperature=0.8)
    st = compare_sequences(out, D, T, None, bk.numpy(), list(range(B)), mode=0, tau=0.8, seed=0,
                           step=0, lam=lam, clip_c=clip_c, grad_seqs=list(range(B)))
    print("sharded clip c=%g: %d band entries, %d compared" % (clip_c, st["clip_band"],
                                                               st["clip_compared"]))
    assert st["clip_compared"] >= 0.99 * (st["clip_compared"] + st["clip_band"])


@pytest.mark.parametrize("V,Pn,align", [(50001, 2, 1), (40000, 2, 8), (151936, 1, 8)])
def test_long_slices_and_workspace_reuse(V, Pn, align):
    # slices of 20000 to 151936 ids (ragged and aligned), then a second step on the same buffers
    B, k = 3, 4
    D, T = rand_case(B, k, k + 1, V, 21, sigma=0.6)
    bk = torch.tensor([4, 2, 3], dtype=torch.int32)
    out, _ = run_sharded(D, T, bk, Pn, align=align, lam=0.5, clip_c=0.2)
    compare_sequences(out, D, T, None, bk.numpy(), list(range(B)), mode=0, tau=1.0, seed=0,
                      step=0, lam=0.5, clip_c=0.2, grad_seqs=[0, 2])
    draft = syn.sample_draft_tokens(D, 1.0, 2)
    out, shards = run_sharded(D, T, bk, Pn, align=align, draft=draft, mode=api.STOCHASTIC,
                              seed=9, step=0, lam=0.5, clip_c=0.2)
    compare_sequences(out, D, T, draft, bk.numpy(), list(range(B)), mode=1, tau=1.0, seed=9,
                      step=0, lam=0.5, clip_c=0.2, grad_seqs=[1])
    # a second step on the same workspaces and exchange buffers
    for s in shards:
        s.set_step(1)
    vp.run_emulated(shards)
    torch.cuda.synchronize()
    assert all(s.device_error() == 0 for s in shards)
    out = dict(shards[0].outputs())
    out["dlogits"] = torch.cat([s.dlogits for s in shards], dim=2)
    compare_sequences(out, D, T, draft, bk.numpy(), list(range(B)), mode=1, tau=1.0, seed=9,
                      step=1, lam=0.5, clip_c=0.2, grad_seqs=[1])


def test_k32_bonus_row_and_verify_only():
    B, k, V = 5, 32, 640
    D, T = rand_case(B, k, k + 1, V, 3, sigma=0.05)   # near-identical rows: long accepted runs
    bk = torch.tensor([32, 32, 1, 17, 31], dtype=torch.int32)
    out, _ = run_sharded(D, T, bk, 4, lam=0.3, clip_c=0.5)
    compare_sequences(out, D, T, None, bk.numpy(), list(range(B)), mode=0, tau=1.0, seed=0,
                      step=0, lam=0.3, clip_c=0.5, grad_seqs=[0, 3])
    draft = syn.sample_draft_tokens(D, 1.0, 4)
    out, _ = run_sharded(D, T, bk, 3, draft=draft, mode=api.STOCHASTIC, seed=5, distill=False)
    compare_sequences(out, D, T, draft, bk.numpy(), list(range(B)), mode=1, tau=1.0, seed=5,
                      step=0, lam=0.3, clip_c=0.5, check_loss=False)


def test_argmax_ties_across_shards():
    # the maximum of every target and draft row appears in two slices: the lowest id wins
    B, k, V = 3, 3, 64
    D = torch.zeros((B, k, V), dtype=torch.bfloat16)
    T = torch.zeros((B, k, V), dtype=torch.bfloat16)
    for b in range(B):
        for i in range(k):
            a, c = 5 + 3 * b + i, 40 + b + i          # slices of 4 ranks: [0,16) [16,32) ...
            T[b, i, a] = T[b, i, c] = 4.0
            D[b, i, c] = D[b, i, a + 16] = 3.0 + 0.5 * (b == 1)
            D[b, i, 2] = -1.0
    bk = torch.full((B,), k, dtype=torch.int32)
    out, _ = run_sharded(D, T, bk, 4, slices=[(0, 16), (16, 16), (32, 16), (48, 16)])
    ri = ri_fields(out["row_info"])
    for b in range(B):
        for i in range(k):
            a, c = 5 + 3 * b + i, 40 + b + i
            assert ri["target_argmax"][b, i] == a
            assert ri["draft_token"][b, i] == min(c, a + 16)
    compare_sequences(out, D, T, None, bk.numpy(), list(range(B)), mode=0, tau=1.0, seed=0,
                      step=0, lam=0.5, clip_c=1.0, grad_seqs=[0, 1, 2])


def test_out_of_range_token_sets_status_on_every_rank():
    B, k, V = 2, 3, 256
    D, T = rand_case(B, k, k, V, 8)
    draft = torch.tensor([[1, 2, 3], [4, V + 5, 6]], dtype=torch.int32)
    bk = torch.full((B,), k, dtype=torch.int32)
    slices = vp.vocab_slices(V, 2)
    shards = [api.VocabShard(D[..., v0:v0 + n].contiguous().cuda(), T[..., v0:v0 + n].contiguous().cuda(),
                             bk.cuda(), V=V, v0=v0, P=2, rank=r, draft_tok=draft.cuda(),
                             mode=api.STOCHASTIC, seed=1) for r, (v0, n) in enumerate(slices)]
    vp.run_emulated(shards)
    torch.cuda.synchronize()
    for s in shards:
        assert s.device_error() == 7                     # SVD_ERR_TOKEN_RANGE
        assert s.device_error() == 0                     # read-and-clear
    assert int(shards[0].accept_len[1]) <= 1             # the bad row counts as rejected


# ------------------------------------------------------------------------------------------
# full-size workloads, sampled sequences
# ------------------------------------------------------------------------------------------
def test_greedy_qwen_b32_eight_shards():
    w = syn.WORKLOADS["greedy_qwen_b32"]
    D, T = syn.make_logits(w)
    h, W1, b1, w2, b2 = syn.make_head(w)
    _, bk = api.svd_length_head(h.cuda(), W1.cuda(), b1.cuda(), w2.cuda(), b2, w.k)
    bk = bk.cpu()
    out, shards = run_sharded(D, T, bk, 8, temperature=w.tau, lam=w.lam, clip_c=w.clip_c)
    seqs = list(range(w.B))
    compare_sequences(out, D, T, None, bk.numpy(), seqs, mode=0, tau=w.tau, seed=0, step=0,
                      lam=w.lam, clip_c=w.clip_c, grad_seqs=[0, 17, 31])
    r = oracle.distill(D, T, bk.numpy(), w.lam, w.clip_c, w.tau, want_grad=False)
    P.assert_close(out["loss_total"].cpu().numpy()[0], r["loss_total"], "loss_total")
    g = out["dlogits"]
    for b in range(w.B):
        n = int(bk[b])
        if n < w.k:
            assert int(torch.count_nonzero(g[b, n:])) == 0


def test_stochastic_qwen_b64_four_shards():
    w = syn.WORKLOADS["stochastic_qwen_b64"]
    D, T = syn.make_logits(w)
    draft = syn.sample_draft_tokens(D, w.tau, 77)
    h, W1, b1, w2, b2 = syn.make_head(w)
    _, bk = api.svd_length_head(h.cuda(), W1.cuda(), b1.cuda(), w2.cuda(), b2, w.k)
    bk = bk.cpu()
    out, _ = run_sharded(D, T, bk, 4, draft=draft, mode=api.STOCHASTIC, temperature=w.tau,
                         seed=w.philox_seed, lam=w.lam, clip_c=w.clip_c)
    st = compare_sequences(out, D, T, draft, bk.numpy(), list(range(w.B)), mode=1, tau=w.tau,
                           seed=w.philox_seed, step=0, lam=w.lam, clip_c=w.clip_c, grad_seqs=[5])
    print("stochastic near-ties:", st)
