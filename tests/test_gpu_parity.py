"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Small cases are compared element by element; the full-size workloads run in the same launch
configuration as the benchmark and are compared on sampled sequences (the oracle regenerates
exactly those sequences on the host) and on the properties that hold at any size.
Tolerances: see tests/parity.py.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verify_distill_b200 import api
from speculative_decoding_verify_distill_b200 import synthetic as syn
from tests import parity as P

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from speculative_decoding_verify_distill_b200 import build
    build.build()
    oracle.build()


def cuda(t):
    return t.to("cuda", non_blocking=False).contiguous()


def ri_fields(ri):
    d = api.row_info_dict(ri.cpu())
    return {k: v.numpy() for k, v in d.items()}


# ------------------------------------------------------------------------------------------
# generic comparison of one fused call against the oracle on a set of sequences
# ------------------------------------------------------------------------------------------
def compare_sequences(out, D, T, draft, bk_used, seqs, *, mode, tau, seed, step, lam, clip_c,
                      grad_scale=1.0, grad_seqs=None, dl_fp32=False, kt=None, check_loss=True):
    """out: dict of GPU outputs (full batch); D, T: host tensors of the sequences `seqs`."""
    n = len(seqs)
    bk_s = bk_used[seqs]
    dr_s = None if draft is None else draft[seqs].numpy()
    ref = oracle.verify(D, T, dr_s, bk_s, mode, tau, seed, step, seq_ids=seqs)
    acc_g = out["accept_len"].cpu().numpy()[seqs]
    em_g = out["emitted"].cpu().numpy()[seqs]
    ne_g = out["n_emitted"].cpu().numpy()[seqs]
    ri = ri_fields(out["row_info"])
    stats = dict(u_ties=0, sample_ties=0, clip_band=0, clip_compared=0)
    k = D.shape[1]
    kt = T.shape[1]
    for j, b in enumerate(seqs):
        nb = int(bk_s[j])
        # per-row: argmax of the target (exact), draft token (exact), lse (tolerance)
        ygpu = ri["target_argmax"][b, :nb]
        assert np.array_equal(ygpu, ref["row_y"][j, :nb]), (b, ygpu, ref["row_y"][j, :nb])
        assert np.array_equal(ri["draft_token"][b, :nb], ref["row_x"][j, :nb]), b
        if nb < kt:
            assert ri["target_argmax"][b, nb] == ref["row_y"][j, nb], b
        tie_seq = False
        if mode == 1:
            acc_gpu = ri["accepted"][b, :nb]
            acc_ref = ref["row_acc"][j, :nb]
            for i in range(nb):
                if acc_gpu[i] != acc_ref[i]:
                    margin = abs(ref["row_u"][j, i] - min(1.0, ref["row_ratio"][j, i]))
                    assert margin < P.TIE_U, (b, i, margin)
                    stats["u_ties"] += 1
                    tie_seq = True
            P.assert_close(ri["ratio"][b, :nb], ref["row_ratio"][j, :nb], "ratio seq %d" % b)
        if tie_seq:
            continue
        assert acc_g[j] == ref["accept_len"][j], (b, acc_g[j], ref["accept_len"][j])
        assert ne_g[j] == ref["n_emitted"][j], b
        if not np.array_equal(em_g[j], ref["emitted"][j]):
            # only the sampled correction / bonus token may differ, and only at a near-tie
            a = int(ref["accept_len"][j])
            diff = np.nonzero(em_g[j] != ref["emitted"][j])[0]
            assert mode == 1 and list(diff) == [a] and ref["fix_margin"][j] < P.TIE_SAMPLE, (
                b, em_g[j], ref["emitted"][j], ref["fix_margin"][j])
            stats["sample_ties"] += 1
    if check_loss:
        want_grad_for = set(grad_seqs or [])
        sub = [j for j, b in enumerate(seqs) if b in want_grad_for]
        r = oracle.distill(D, T, bk_s, lam, clip_c, tau, grad_scale, want_grad=False)
        # clip decisions fp32 cannot fix: counted entries, bounded effect on the row sums
        cb = P.clip_band(D, T, bk_s, clip_c, tau, want_mask=bool(sub))
        stats["clip_band"] = int(cb["n_band"].sum())
        stats["clip_compared"] = int(bk_s.sum()) * D.shape[2] - stats["clip_band"]
        lr_g = out["loss_rows"].cpu().numpy()[seqs]
        P.assert_close(lr_g, r["loss_rows"], "loss_rows", extra=(1.0 - lam) * cb["dK"])
        verified = np.arange(k)[None, :] < bk_s[:, None]
        lse_g = ri["lse_draft"][seqs][:, :k]
        P.assert_close(lse_g[verified], _oracle_lse(D, bk_s, tau)[verified], "lse_draft")
        for j in sub:
            b = seqs[j]
            rg = oracle.distill(D[j:j + 1], T[j:j + 1], bk_s[j:j + 1], lam, clip_c, tau, grad_scale)
            g = out["dlogits"][b].cpu()
            keep = ~cb["band"][j]
            extra = None
            if cb["n_band"][j].any():
                q = P.softmax_rows(D[j], tau)
                extra = (grad_scale / tau) * (1.0 - lam) * q * cb["dS"][j][:, None]
            if dl_fp32:
                P.assert_close(g.numpy(), rg["dlogits"][0], "dlogits fp32 seq %d" % b, mask=keep,
                               extra=extra)
            else:
                P.assert_bf16_grad(g, rg["dlogits"][0], "dlogits bf16 seq %d" % b, mask=keep,
                                   extra=extra)
    return stats


def _oracle_lse(D, bk, tau):
    B, k, V = D.shape
    out = np.full((B, k), np.nan)
    for b in range(B):
        for i in range(int(bk[b])):
            out[b, i] = oracle.row_stats(D[b, i], tau)[2]
    return out


def run_fused(w: syn.Workload, D, T, *, draft=None, use_head=True, bk_in=None, lam=None, clip_c=None,
              tau=None, dl_fp32=False, grad_scale=1.0, step=0, kt_override=None):
    lam = w.lam if lam is None else lam
    clip_c = w.clip_c if clip_c is None else clip_c
    tau = w.tau if tau is None else tau
    head = None
    if use_head:
        h, W1, b1, w2, b2 = syn.make_head(w)
        head = (cuda(h), cuda(W1), cuda(b1), cuda(w2), b2)
    vd = api.VerifyDistill(cuda(D), cuda(T), head=head, bk_in=None if bk_in is None else cuda(bk_in),
                           draft_tok=None if draft is None else cuda(draft), mode=w.mode,
                           temperature=tau, seed=w.philox_seed, step=step, lam=lam, clip_c=clip_c,
                           grad_scale=grad_scale, dlogits_fp32=dl_fp32, row_info=True)
    vd()
    torch.cuda.synchronize()
    assert api.svd_get_device_error(vd.ws) == 0
    return vd.outputs()


def check_bk(out, w: syn.Workload):
    """b_k bit-exact against the oracle except at counted near-integers of gamma*bhat*k, which
    must stay rare (at most 1% of the batch, and at least one allowed)."""
    h, W1, b1, w2, b2 = syn.make_head(w)
    bhat_ref, bk_ref, _ = oracle.length_head(h, W1, b1, w2, b2, w.k, 1.0, 0)
    bk_gpu = out["bk"].cpu().numpy()
    bhat_gpu = out["bhat"].cpu().numpy()
    near = P.bk_near_integer(bhat_ref, w.k)
    n_near = int(near.sum())
    print("%s: b_k near an integer (excluded from the exact check): %d of %d" % (w.name, n_near, w.B))
    assert n_near <= max(1, w.B // 100), n_near
    assert np.array_equal(bk_gpu[~near], bk_ref[~near])
    P.assert_close(bhat_gpu, bhat_ref, "bhat", rtol=1e-4, atol=1e-6)
    return bk_gpu, n_near


# ------------------------------------------------------------------------------------------
# the five workloads
# ------------------------------------------------------------------------------------------
def test_tiny_full_parity():
    w = syn.WORKLOADS["tiny"]
    D, T = syn.make_logits(w)
    for dl32 in (False, True):
        out = run_fused(w, D, T, dl_fp32=dl32)
        bk, _ = check_bk(out, w)
        seqs = list(range(w.B))
        compare_sequences(out, D, T, None, bk, seqs, mode=0, tau=w.tau, seed=0, step=0,
                          lam=w.lam, clip_c=w.clip_c, grad_seqs=seqs, dl_fp32=dl32)
        r = oracle.distill(D, T, bk, w.lam, w.clip_c, w.tau, want_grad=False)
        P.assert_close(out["loss_total"].cpu().numpy()[0], r["loss_total"], "loss_total")


def test_greedy_qwen_b32_sampled():
    w = syn.WORKLOADS["greedy_qwen_b32"]
    D, T = syn.make_logits(w)
    out = run_fused(w, D, T)
    bk, _ = check_bk(out, w)
    seqs = list(range(w.B))
    compare_sequences(out, D, T, None, bk, seqs, mode=0, tau=w.tau, seed=0, step=0, lam=w.lam,
                      clip_c=w.clip_c, grad_seqs=[0, 17, 31])
    r = oracle.distill(D, T, bk, w.lam, w.clip_c, w.tau, want_grad=False)
    P.assert_close(out["loss_total"].cpu().numpy()[0], r["loss_total"], "loss_total")


def test_ragged_qwen_b128_sampled():
    w = syn.WORKLOADS["ragged_qwen_b128"]
    D, T = syn.make_logits(w)
    out = run_fused(w, D, T)
    bk, _ = check_bk(out, w)
    assert len(set(bk.tolist())) >= 8, np.bincount(bk)      # ragged verification lengths
    order = np.argsort(bk)
    seqs = sorted(set(order[:6].tolist() + order[-6:].tolist() + list(range(0, w.B, 16))))
    Ds, Ts = D[seqs], T[seqs]
    compare_sequences(out, Ds, Ts, None, bk, seqs, mode=0, tau=w.tau, seed=0, step=0, lam=w.lam,
                      clip_c=w.clip_c, grad_seqs=[int(order[0]), int(order[-1]), seqs[3]])
    # properties at full size: zero gradient rows beyond b_k, accepted <= b_k
    g = out["dlogits"]
    for b in range(0, w.B, 7):
        n = int(bk[b])
        if n < w.k:
            assert int(torch.count_nonzero(g[b, n:])) == 0
    assert (out["accept_len"].cpu().numpy() <= bk).all()


def test_stochastic_qwen_b64_sampled():
    w = syn.WORKLOADS["stochastic_qwen_b64"]
    D, T = syn.make_logits(w)
    draft = syn.sample_draft_tokens(D, w.tau, 77)
    out = run_fused(w, D, T, draft=draft)
    bk, _ = check_bk(out, w)
    seqs = list(range(w.B))
    st = compare_sequences(out, D, T, draft, bk, seqs, mode=1, tau=w.tau, seed=w.philox_seed,
                           step=0, lam=w.lam, clip_c=w.clip_c, grad_seqs=[5])
    print("stochastic near-ties:", st)
    check_sample_rows(out, w)
    # the same workload with every b_k = k (full verification)
    out2 = run_fused(w, D, T, draft=draft, use_head=False, bk_in=torch.full((w.B,), w.k, dtype=torch.int32))
    compare_sequences(out2, D[:16], T[:16], draft, np.full(w.B, w.k, np.int32), seqs[:16], mode=1,
                      tau=w.tau, seed=w.philox_seed, step=0, lam=w.lam, clip_c=w.clip_c,
                      check_loss=False)


def check_sample_rows(out, w):
    """Stochastic rows: the drawn token sits on the row it was drawn from (the first rejected
    row, else the bonus row) and equals the emitted one; every other row reports none."""
    ri = ri_fields(out["row_info"])
    acc = out["accept_len"].cpu().numpy()
    bk = out["bk"].cpu().numpy()
    em = out["emitted"].cpu().numpy()
    for b in range(w.B):
        a, nb = int(acc[b]), int(bk[b])
        s = ri["sample_token"][b].copy()
        if a < nb or nb < s.shape[0]:
            assert s[a] == em[b, a] and 0 <= s[a] < w.V, (b, a, s[a], em[b, a])
            s[a] = -1
        assert (s == -1).all(), (b, a, ri["sample_token"][b])


@pytest.mark.parametrize("clip_c,lam", syn.STRESS_SWEEP)
def test_stress_llama_b256_sweep(clip_c, lam, _stress_inputs):
    w = syn.WORKLOADS["stress_llama_b256"]
    D, T = _stress_inputs
    out = run_fused(w, D, T, lam=lam, clip_c=clip_c)
    bk, _ = check_bk(out, w)
    seqs = [3, 128, 255]
    compare_sequences(out, D[seqs], T[seqs], None, bk, seqs, mode=0, tau=w.tau, seed=0, step=0,
                      lam=lam, clip_c=clip_c, grad_seqs=[128])


@pytest.fixture(scope="module")
def _stress_inputs():
    return syn.make_logits(syn.WORKLOADS["stress_llama_b256"])


def test_emission_law_v8_million_trials():
    # 10^6 independent trials of one draft position at V = 8: emitted tokens follow p
    N, V = 1_000_000, 8
    d_row = np.array([2.0, 1.0, 0.5, 0.0, -1.0, 1.5, 0.25, -0.5], np.float32)
    t_row = np.array([0.5, 1.5, 0.0, 1.0, 0.5, -1.0, 0.75, 0.0], np.float32)
    D = torch.from_numpy(np.broadcast_to(d_row, (N, 1, V)).copy()).to(torch.bfloat16)
    T = torch.from_numpy(np.broadcast_to(t_row, (N, 1, V)).copy()).to(torch.bfloat16)
    draft = syn.sample_draft_tokens_batched(D, 1.0, 17)
    bk = torch.ones(N, dtype=torch.int32)
    out = api.svd_verify(cuda(D), cuda(T), cuda(draft), cuda(bk), api.STOCHASTIC, 1.0, 1234, 0)
    tok = out["emitted"][:, 0].cpu().numpy()
    counts = np.bincount(tok, minlength=V)
    p = torch.softmax(torch.from_numpy(t_row).to(torch.bfloat16).double(), 0).numpy()
    chi2 = (((counts - N * p) ** 2) / (N * p)).sum()
    import scipy.stats
    assert chi2 < scipy.stats.chi2.ppf(1 - 1e-4, V - 1), (chi2, counts, N * p)
    # bit-level agreement with the oracle on the first 20000 trials
    n = 20_000
    ref = oracle.verify(D[:n], T[:n], draft[:n].numpy(), bk[:n].numpy(), 1, 1.0, 1234, 0)
    g_acc = out["accept_len"].cpu().numpy()[:n]
    mism = np.nonzero(g_acc != ref["accept_len"])[0]
    for j in mism:
        assert abs(ref["row_u"][j, 0] - min(1.0, ref["row_ratio"][j, 0])) < P.TIE_U
    ok = np.ones(n, bool)
    ok[mism] = False
    differ = ok & (tok[:n] != ref["emitted"][:, 0])
    assert (ref["fix_margin"][differ] < P.TIE_SAMPLE).all(), np.nonzero(differ)[0][:10]
