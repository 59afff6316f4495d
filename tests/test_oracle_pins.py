"""Pins of the CPU oracle to things other than itself (CPU only).

Each test ties one oracle function to a library routine, a closed form, an invariant the pages
or the mathematics fix, or brute force on tiny inputs, chosen so that a dropped term, a wrong
sign/index or a transposed operand fails at least one of them.
"""
import json
import math
import os
import sys

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch
import torch.nn.functional as F

from speculative_decoding_verify_distill_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def f64(t):
    return t.to(torch.float64).numpy()


# ------------------------------------------------------------------------------------------
# a2: row statistics
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("V", [1, 8, 1024])
@pytest.mark.parametrize("tau", [1.0, 0.7])
def test_row_stats_vs_scipy_and_numpy(orc, V, tau):
    g = torch.Generator().manual_seed(V)
    for trial in range(20):
        x = bf16(3 * torch.randn(V, generator=g).numpy())
        mx, am, lse = orc.row_stats(x, tau)
        xd = f64(x)
        assert mx == xd.max()
        assert am == int(np.argmax(xd))          # numpy returns the first maximal index
        assert lse == pytest.approx(scipy.special.logsumexp(xd / tau), rel=1e-14, abs=1e-14)


def test_argmax_ties_take_lowest_id(orc):
    for V, ids in [(8, [2, 5]), (8, [0, 7]), (1024, [3, 500, 1023]), (1024, [1023])]:
        x = np.full(V, -1.0, np.float32)
        x[ids] = 7.25                             # exactly representable in bf16
        mx, am, _ = orc.row_stats(bf16(x))
        assert (mx, am) == (7.25, min(ids))


def test_row_stats_bruteforce_v8(orc):
    # every value drawn from a 4-point grid: many exact ties, lse by direct enumeration
    rng = np.random.default_rng(0)
    for _ in range(200):
        x = rng.choice([-2.0, 0.0, 0.5, 3.0], size=8).astype(np.float32)
        _, am, lse = orc.row_stats(bf16(x))
        best = max(range(8), key=lambda v: (x[v], -v))
        assert am == best
        assert lse == pytest.approx(math.log(sum(math.exp(float(t)) for t in x)), rel=1e-14)


# ------------------------------------------------------------------------------------------
# a1: length head
# ------------------------------------------------------------------------------------------
def test_length_head_vs_torch_linear(orc):
    w = syn.WORKLOADS["tiny"]
    h, W1, b1, w2, b2 = syn.make_head(w)
    b1 = torch.linspace(-0.1, 0.1, w.M)            # non-zero bias to exercise that term
    bhat, bk, z = orc.length_head(h, W1, b1, w2, 0.03, w.k)
    hid = F.relu(F.linear(h.double(), W1.double(), b1.double()))
    zt = hid @ w2.double() + 0.03
    assert np.allclose(z, zt.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(bhat, torch.sigmoid(zt).numpy(), rtol=1e-12, atol=1e-14)
    assert bk.min() >= 1 and bk.max() <= w.k


def test_length_head_bk_edges(orc):
    # zero weights: hidden = 0, z = b2, bhat = sigmoid(b2)
    H, M, k = 16, 4, 8
    h = bf16(np.ones((3, H)))
    W1 = bf16(np.zeros((M, H)))
    w2 = bf16(np.zeros(M))
    cases = [  # (b2, gamma, ceil result, floor result)
        (0.0, 1.0, 4, 4),          # bhat = 1/2, bhat*k = 4 exactly: ceil == floor
        (0.01, 1.0, 5, 4),         # bhat*k = 4.02
        (-0.01, 1.0, 4, 3),        # bhat*k = 3.98
        (-60.0, 1.0, 1, 1),        # bhat -> 0: clamped up to 1
        (60.0, 1.0, 8, 8),         # bhat -> 1: k
        (0.0, 2.0, 8, 8),          # gamma * bhat * k = 8
        (0.0, 3.0, 8, 8),          # 12 clamped to k
        (0.0, 0.1, 1, 1),          # 0.4: ceil 1, floor 0 -> clamp 1
    ]
    for b2, gamma, want_ceil, want_floor in cases:
        _, bkc, _ = orc.length_head(h, W1, None, w2, b2, k, gamma, 0)
        _, bkf, _ = orc.length_head(h, W1, None, w2, b2, k, gamma, 1)
        assert list(bkc) == [want_ceil] * 3, (b2, gamma)
        assert list(bkf) == [want_floor] * 3, (b2, gamma)


# ------------------------------------------------------------------------------------------
# a5: loss and gradient
# ------------------------------------------------------------------------------------------
def test_closed_forms(orc):
    with open(os.path.join(GOLDEN, "closed_forms.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        D = np.asarray(c["D"], np.float64).reshape(1, 1, -1)
        T = np.asarray(c["T"], np.float64).reshape(1, 1, -1)
        clip = math.inf if c["clip_c"] == "inf" else c["clip_c"]
        r = orc.distill(D, T, [1], c["lam"], clip, c["tau"])
        assert r["loss_rows"][0, 0] == pytest.approx(c["loss"], abs=1e-13), c["name"]
        assert r["rkl_rows"][0, 0] == pytest.approx(c["rkl"], abs=1e-13), c["name"]
        assert r["kc_rows"][0, 0] == pytest.approx(c["kc"], abs=1e-13), c["name"]
        assert r["ce_rows"][0, 0] == pytest.approx(c["ce"], abs=1e-13), c["name"]
        assert np.allclose(r["dlogits"][0, 0], c["grad"], atol=1e-13), c["name"]
        # the same case through the bf16 entry point (all inputs are exact in bf16)
        rb = orc.distill(bf16(D), bf16(T), [1], c["lam"], clip, c["tau"])
        assert rb["loss_rows"][0, 0] == pytest.approx(c["loss"], abs=1e-13)


def _rand_rows(seed, B, k, V, sigma=0.7, kt=None):
    g = torch.Generator().manual_seed(seed)
    kt = kt or k
    T = 2 * torch.randn(B, kt, V, generator=g)
    D = T[:, :k] + sigma * torch.randn(B, k, V, generator=g)
    return D.to(torch.bfloat16), T.to(torch.bfloat16)


def test_loss_equal_rows_is_pure_ce(orc):
    D, _ = _rand_rows(1, 3, 4, 64)
    r = orc.distill(D, D, [4, 4, 4], 0.3, 0.01)
    assert np.abs(r["rkl_rows"]).max() < 1e-15
    assert np.abs(r["kc_rows"]).max() < 1e-15
    assert np.allclose(r["loss_rows"], 0.3 * r["ce_rows"], rtol=1e-14)


def test_lambda_one_is_cross_entropy(orc):
    D, T = _rand_rows(2, 3, 4, 257)
    for tau in (1.0, 0.5):
        r = orc.distill(D, T, [4, 4, 4], 1.0, 0.1, tau)
        y = T.double().argmax(-1)                   # torch argmax: first maximal index
        ce = F.cross_entropy((D.double() / tau).reshape(-1, 257), y.reshape(-1),
                             reduction="none").reshape(3, 4)
        assert np.allclose(r["loss_rows"], ce.numpy(), rtol=1e-12, atol=1e-12)
        assert r["loss_total"] == pytest.approx(float(ce.sum()), rel=1e-12)


def test_lambda_zero_unclipped_is_kl_div(orc):
    D, T = _rand_rows(3, 2, 5, 300)
    for tau in (1.0, 1.7):
        r = orc.distill(D, T, [5, 5], 0.0, math.inf, tau)
        lq = F.log_softmax(D.double() / tau, -1)
        lp = F.log_softmax(T.double() / tau, -1)
        # kl_div(input=log p, target=log q, log_target) = sum q (log q - log p): reverse KL
        kl = F.kl_div(lp, lq, reduction="none", log_target=True).sum(-1)
        assert np.allclose(r["loss_rows"], kl.numpy(), rtol=1e-11, atol=1e-13)
        assert (r["rkl_rows"] >= 0).all()


def test_clipping_invariants(orc):
    D, T = _rand_rows(4, 2, 6, 128, sigma=1.5)
    bk = [6, 6]
    prev = None
    rk = orc.distill(D, T, bk, 0.0, math.inf)["rkl_rows"]
    for c in (0.0, 0.001, 0.01, 0.1, 1.0, 10.0, 1e9):
        r = orc.distill(D, T, bk, 0.0, c)
        assert (r["kc_rows"] <= r["rkl_rows"] + 1e-15).all()
        assert np.allclose(r["rkl_rows"], rk, rtol=1e-14)
        if prev is not None:
            assert (r["kc_rows"] >= prev - 1e-15).all()   # K_c is non-decreasing in c
        prev = r["kc_rows"]
    assert np.allclose(prev, rk, rtol=1e-14)                  # c beyond every entry: plain RKL


def test_clip_band_special_cases(orc):
    """The parity band of the clip decision (entries with |d_v - c| < eps q_v (1 + |s_v|)),
    pinned on cases whose d_v are known in closed form."""
    # D = [0, 0], T = [1, 0]: q = (1/2, 1/2), s1 = log((1 + e)/2), d1 = s1 / 2 (hand-derived)
    e = math.e
    s1 = math.log((1 + e) / 2)
    d1 = s1 / 2
    D = bf16(np.array([0.0, 0.0]).reshape(1, 1, 2))
    T = bf16(np.array([1.0, 0.0]).reshape(1, 1, 2))
    cb = orc.clip_band(D, T, [1], d1, 1.0, 2e-5)
    assert cb["n_band"].tolist() == [[1]] and cb["band"][0, 0].tolist() == [False, True]
    assert cb["dS"][0, 0] == pytest.approx(0.5 * abs(s1 + 1), rel=1e-12)
    assert cb["dK"][0, 0] < 1e-15
    for c in (d1 * (1 + 1e-3), d1 * (1 - 1e-3), 0.0, math.inf):
        assert orc.clip_band(D, T, [1], c, 1.0, 2e-5)["n_band"][0, 0] == 0, c
    assert orc.clip_band(D, T, [1], d1, 1.0, 0.0)["n_band"][0, 0] == 0   # empty band
    # D = T: every s_v = 0, so at c = 0 every entry lies on the boundary; S moves by sum q = 1
    Dq, _ = _rand_rows(11, 2, 3, 97)
    cb = orc.clip_band(Dq, Dq, [3, 1], 0.0, 0.8, 2e-5)
    assert cb["n_band"].tolist() == [[97, 97, 97], [97, 0, 0]]      # rows past b_k have none
    assert np.allclose(cb["dS"][0], 1.0, rtol=1e-12) and cb["dS"][1, 1:].max() == 0.0
    assert cb["dK"].max() == 0.0
    assert orc.clip_band(Dq, Dq, [3, 1], 1e-3, 0.8, 2e-5)["n_band"].max() == 0


def test_clip_band_brackets_decision_flips(orc):
    """An entry whose d_v equals c (fp64, computed here by torch) is in the band of its row."""
    D, T = _rand_rows(12, 2, 4, 512, sigma=2.0)
    bk = [4, 3]
    lq = F.log_softmax(D.double(), -1).numpy()
    lp = F.log_softmax(T.double(), -1).numpy()
    d = np.exp(lq) * (lq - lp)
    for b, n in enumerate(bk):
        for i in range(n):
            c = float(np.sort(d[b, i])[-3])          # an entry sits exactly on the clip bound
            cb = orc.clip_band(D[b:b + 1, i:i + 1], T[b:b + 1, i:i + 1], [1], c, 1.0, 2e-5)
            v = int(np.argmax(d[b, i] == c))
            assert cb["band"][0, 0, v]
            assert cb["n_band"][0, 0] >= 1


def test_rows_beyond_bk_are_zero(orc):
    D, T = _rand_rows(5, 3, 6, 50)
    bk = [1, 3, 6]
    r = orc.distill(D, T, bk, 0.5, 1.0)
    full = orc.distill(D, T, [6, 6, 6], 0.5, 1.0)
    for b, n in enumerate(bk):
        assert (r["loss_rows"][b, n:] == 0).all()
        assert (r["dlogits"][b, n:] == 0).all()
        assert np.array_equal(r["loss_rows"][b, :n], full["loss_rows"][b, :n])
        assert np.array_equal(r["dlogits"][b, :n], full["dlogits"][b, :n])
    assert r["loss_total"] == pytest.approx(sum(r["loss_rows"][b, :n].sum() for b, n in enumerate(bk)))


def test_kt_plus_one_uses_matching_target_rows(orc):
    D, T = _rand_rows(6, 2, 4, 40, kt=5)
    r = orc.distill(D, T, [4, 2], 0.5, 0.2)
    r2 = orc.distill(D, T[:, :4].contiguous(), [4, 2], 0.5, 0.2)
    assert np.array_equal(r["dlogits"], r2["dlogits"])


def _torch_loss(Dd, Td, lam, c, tau, y):
    """Independent restatement of the loss for autograd: torch softmax, clamp, gather."""
    lq = F.log_softmax(Dd / tau, -1)
    lp = F.log_softmax(Td / tau, -1)
    q = lq.exp()
    d = q * (lq - lp)
    kc = torch.clamp(d, max=c).sum(-1)
    ce = -lq.gather(-1, y.unsqueeze(-1)).squeeze(-1)
    return (lam * ce + (1 - lam) * kc).sum()


def _far_from_clip(Dd, Td, c, tau, gap):
    lq = F.log_softmax(Dd / tau, -1)
    lp = F.log_softmax(Td / tau, -1)
    d = lq.exp() * (lq - lp)
    return bool(((d - c).abs() > gap).all())


@pytest.mark.parametrize("V", [8, 1024])
@pytest.mark.parametrize("lam,c,tau", [(0.5, 1.0, 1.0), (0.0, 0.05, 1.0), (1.0, 0.1, 1.0),
                                       (0.8, 0.01, 0.7), (0.3, math.inf, 2.0)])
def test_gradient_autograd(orc, V, lam, c, tau):
    g = torch.Generator().manual_seed(V + int(100 * lam))
    Dd = (2 * torch.randn(2, 3, V, generator=g, dtype=torch.float64))
    Td = Dd + 1.2 * torch.randn(2, 3, V, generator=g, dtype=torch.float64)
    if V == 8:
        Dd[0, 0, 3] = Dd[0, 0].max() + 3.0             # a confident draft: clipping kicks in
    r = orc.distill(Dd.numpy(), Td.numpy(), [3, 3], lam, c, tau, grad_scale=0.25)
    Dg = Dd.clone().requires_grad_(True)
    y = Td.argmax(-1)
    loss = _torch_loss(Dg, Td, lam, c, tau, y)
    loss.backward()
    assert r["loss_total"] == pytest.approx(float(loss.detach()), rel=1e-12, abs=1e-12)
    assert np.allclose(r["dlogits"], 0.25 * Dg.grad.numpy(), rtol=1e-9, atol=1e-13)
    # the gradient of a softmax-based loss sums to zero over the vocabulary
    assert np.abs(r["dlogits"].sum(-1)).max() < 1e-12


@pytest.mark.parametrize("V", [8, 1024])
def test_gradient_finite_differences(orc, V):
    g = torch.Generator().manual_seed(11 * V)
    Dd = 2 * torch.randn(1, 1, V, generator=g, dtype=torch.float64)
    Td = Dd + 0.9 * torch.randn(1, 1, V, generator=g, dtype=torch.float64)
    Dd[0, 0, 1] += 4.0
    lam, c, tau, h = 0.4, 0.05, 1.3, 1e-6
    assert _far_from_clip(Dd, Td, c, tau, 1e-4)
    r = orc.distill(Dd.numpy(), Td.numpy(), [1], lam, c, tau)
    idx = range(V) if V <= 8 else list(range(0, V, 37)) + [1, int(Td.argmax())]
    for u in idx:
        Dp = Dd.clone(); Dp[0, 0, u] += h
        Dm = Dd.clone(); Dm[0, 0, u] -= h
        if not (_far_from_clip(Dp, Td, c, tau, 1e-5) and _far_from_clip(Dm, Td, c, tau, 1e-5)):
            continue
        lp_ = orc.distill(Dp.numpy(), Td.numpy(), [1], lam, c, tau, want_grad=False)["loss_total"]
        lm_ = orc.distill(Dm.numpy(), Td.numpy(), [1], lam, c, tau, want_grad=False)["loss_total"]
        fd = (lp_ - lm_) / (2 * h)
        assert r["dlogits"][0, 0, u] == pytest.approx(fd, rel=1e-5, abs=1e-8), u


# ------------------------------------------------------------------------------------------
# a3/a4: acceptance and emission
# ------------------------------------------------------------------------------------------
def test_greedy_draft_equals_target_accepts_all(orc):
    D, _ = _rand_rows(7, 5, 6, 100)
    bk = [1, 2, 4, 6, 6]
    r = orc.verify(D, D.clone(), None, bk, 0)
    assert list(r["accept_len"]) == bk
    am = D.double().argmax(-1).numpy()
    for b, n in enumerate(bk):
        # no bonus row when kt == k and all k are accepted; otherwise the bonus is argmax T_n
        want = list(am[b, :n]) + ([am[b, n]] if n < 6 else [])
        assert list(r["emitted"][b, :len(want)]) == want
        assert (r["emitted"][b, len(want):] == -1).all()
        assert r["n_emitted"][b] == len(want)


def test_greedy_handbuilt_mismatches(orc):
    V, k = 8, 4
    D = np.zeros((1, k, V), np.float32)
    T = np.zeros((1, k + 1, V), np.float32)
    draft_arg = [3, 1, 6, 2]
    target_arg = [3, 1, 5, 2, 7]
    for i in range(k):
        D[0, i, draft_arg[i]] = 2.0
    for i in range(k + 1):
        T[0, i, target_arg[i]] = 2.0
    for n, acc, emitted in [(4, 2, [3, 1, 5]), (2, 2, [3, 1, 5]), (1, 1, [3, 1]),
                            (3, 2, [3, 1, 5])]:
        r = orc.verify(bf16(D), bf16(T), None, [n], 0)
        assert r["accept_len"][0] == acc
        assert list(r["emitted"][0, : len(emitted)]) == emitted
        assert r["n_emitted"][0] == len(emitted)
    # position 2 fixed: everything accepted, bonus from target row 4 (kt = k + 1)
    D[0, 2] = 0; D[0, 2, 5] = 2.0
    r = orc.verify(bf16(D), bf16(T), None, [4], 0)
    assert r["accept_len"][0] == 4 and list(r["emitted"][0]) == [3, 1, 5, 2, 7]
    # caller-provided draft tokens override the draft argmax
    r = orc.verify(bf16(D), bf16(T), np.array([[3, 0, 5, 2]]), [4], 0)
    assert r["accept_len"][0] == 1 and list(r["emitted"][0, :2]) == [3, 1]


def test_stochastic_q_equals_p_accepts_all(orc):
    D, _ = _rand_rows(8, 16, 5, 64)
    x = syn.sample_draft_tokens_batched(D, 1.0, 3)
    r = orc.verify(D, D.clone(), x, [5] * 16, 1, 1.0, seed=99, step=4)
    assert (r["accept_len"] == 5).all()
    assert np.allclose(r["row_ratio"], 1.0, rtol=1e-12)


def _softmax(x):
    e = np.exp(x - x.max())
    return e / e.sum()


def test_emission_law_matches_target_v8(orc):
    # Speculative sampling emits each token with probability exactly p_v.  One draft position,
    # N independent trials (each its own sequence index, hence its own Philox counters).
    N, V = 400_000, 8
    d_row = np.array([2.0, 1.0, 0.5, 0.0, -1.0, 1.5, 0.25, -0.5], np.float32)
    t_row = np.array([0.5, 1.5, 0.0, 1.0, 0.5, -1.0, 0.75, 0.0], np.float32)
    D = bf16(np.broadcast_to(d_row, (N, 1, V)).copy())
    T = bf16(np.broadcast_to(t_row, (N, 1, V)).copy())
    x = syn.sample_draft_tokens_batched(D, 1.0, 17)
    r = orc.verify(D, T, x, np.ones(N, np.int32), 1, 1.0, seed=1234, step=0)
    tok = r["emitted"][:, 0]
    counts = np.bincount(tok, minlength=V)
    p = _softmax(f64(bf16(t_row)))
    chi2 = (((counts - N * p) ** 2) / (N * p)).sum()
    assert chi2 < scipy.stats.chi2.ppf(1 - 1e-4, V - 1), (chi2, counts, N * p)
    # a rejected draft is always followed by a residual token different in law from q
    q = _softmax(f64(bf16(d_row)))
    chi2_q = (((counts - N * q) ** 2) / (N * q)).sum()
    assert chi2_q > 1000


def test_expected_tokens_closed_form(orc):
    # Referee minor comment 1 (their Eq. 1): with the same (p, q) at every position and the bonus
    # row present (kt = k + 1), emitted tokens per step average (1 - A^(k+1)) / (1 - A),
    # A = sum_v min(p_v, q_v).
    N, k, V = 60_000, 4, 8
    d_row = np.array([1.0, 0.5, 0.0, -0.5, 2.0, 0.0, 0.25, -1.0], np.float32)
    t_row = np.array([0.5, 1.0, 0.0, 0.0, 1.0, 0.5, -0.25, 0.0], np.float32)
    D = bf16(np.broadcast_to(d_row, (N, k, V)).copy())
    T = bf16(np.broadcast_to(t_row, (N, k + 1, V)).copy())
    x = syn.sample_draft_tokens_batched(D, 1.0, 5)
    r = orc.verify(D, T, x, np.full(N, k, np.int32), 1, 1.0, seed=7, step=3)
    p, q = _softmax(f64(bf16(t_row))), _softmax(f64(bf16(d_row)))
    A = np.minimum(p, q).sum()
    want = orc.expected_tokens(A, k)
    assert want == pytest.approx(sum(A ** j for j in range(k + 1)), rel=1e-12)
    ne = r["n_emitted"].astype(np.float64)
    se = ne.std() / math.sqrt(N)
    assert abs(ne.mean() - want) < 5 * se, (ne.mean(), want, se)


def test_expected_tokens_special_values(orc):
    assert orc.expected_tokens(0.0, 7) == 1.0
    assert orc.expected_tokens(1.0, 7) == 8.0
    assert orc.expected_tokens(0.5, 4) == pytest.approx(1.9375)


def test_inverse_cdf_bruteforce(orc):
    rng = np.random.default_rng(3)
    for _ in range(300):
        V = int(rng.integers(1, 9))
        w = rng.choice([0.0, 0.125, 0.25, 1.0, 3.0], size=V)
        if w.sum() == 0:
            assert orc.sample_inverse_cdf(w, 0.5)[0] == -1
            continue
        u = float(rng.random())
        tok, _ = orc.sample_inverse_cdf(w, u)
        t = u * w.sum()
        want = next(v for v in range(V) if w[: v + 1].sum() > t)
        assert tok == want
        assert w[tok] > 0


def test_out_of_range_draft_token_is_reported(orc):
    D, T = _rand_rows(9, 1, 2, 16)
    r = orc.verify(D, T, np.array([[3, 16]]), [2], 1)
    assert r["token_error"]


# ------------------------------------------------------------------------------------------
# Philox4x32-10
# ------------------------------------------------------------------------------------------
def test_philox_uniformity_and_independence(orc):
    words = np.array([orc.philox_words(1234, 0, s, p) for s in range(64) for p in range(32)],
                     dtype=np.uint64)
    assert len({tuple(w) for w in words.tolist()}) == words.shape[0]
    for j in range(4):
        u = (words[:, j] >> np.uint64(8)).astype(np.float64) / 2 ** 24
        counts = np.histogram(u, bins=16, range=(0, 1))[0]
        chi2 = ((counts - u.size / 16) ** 2 / (u.size / 16)).sum()
        assert chi2 < scipy.stats.chi2.ppf(1 - 1e-4, 15)
    # bit balance of every output bit
    bits = np.unpackbits(words.astype(">u4").view(np.uint8)).reshape(words.shape[0], -1)
    frac = bits.mean(0)
    assert np.abs(frac - 0.5).max() < 0.06


def test_philox_avalanche(orc):
    rng = np.random.default_rng(5)
    flips = []
    for _ in range(200):
        ctr = rng.integers(0, 2 ** 32, 4, dtype=np.uint64).astype(np.uint32)
        key = rng.integers(0, 2 ** 32, 2, dtype=np.uint64).astype(np.uint32)
        a = orc.philox4x32_10(ctr, key)
        c2 = ctr.copy()
        c2[int(rng.integers(0, 4))] ^= np.uint32(1 << int(rng.integers(0, 32)))
        b = orc.philox4x32_10(c2, key)
        flips.append(sum(bin(int(x) ^ int(y)).count("1") for x, y in zip(a, b)))
    assert 60 < np.mean(flips) < 68      # ~64 of 128 output bits change


def test_philox_words_layout(orc):
    # counter = (pos, seq, step_lo, step_hi), key = (seed_lo, seed_hi)
    seed, step = (7 << 32) | 99, (3 << 32) | 5
    w = orc.philox_words(seed, step, 11, 2)
    ref = orc.philox4x32_10([2, 11, 5, 3], [99, 7])
    assert np.array_equal(w, ref)


def test_philox_key_avalanche(orc):
    # every key bit must reach the output: flipping one changes about half of the 128 bits
    rng = np.random.default_rng(6)
    for word in (0, 1):
        flips = []
        for _ in range(100):
            ctr = rng.integers(0, 2 ** 32, 4, dtype=np.uint64).astype(np.uint32)
            key = rng.integers(0, 2 ** 32, 2, dtype=np.uint64).astype(np.uint32)
            k2 = key.copy()
            k2[word] ^= np.uint32(1 << int(rng.integers(0, 32)))
            a, b = orc.philox4x32_10(ctr, key), orc.philox4x32_10(ctr, k2)
            flips.append(sum(bin(int(x) ^ int(y)).count("1") for x, y in zip(a, b)))
        assert 60 < np.mean(flips) < 68, word


def _curand_host_lib():
    """libcurand (the CUDA toolkit's, or the one that ships with torch); None if absent."""
    import ctypes
    import glob
    import os
    cands = [os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "lib64", "libcurand.so")]
    for sp in sys.path:
        cands += sorted(glob.glob(os.path.join(sp, "nvidia", "curand", "lib", "libcurand.so*")))
    for c in cands:
        if os.path.exists(c):
            try:
                return ctypes.CDLL(c)
            except OSError:
                continue
    return None


def _curand_host_philox_blocks(lib, seed, first_block, nblocks):
    """Raw 32-bit outputs of cuRAND's host-side Philox4x32-10 generator (public API, no GPU),
    from output 4 * first_block on, as [nblocks, 4]."""
    import ctypes
    gen = ctypes.c_void_p()
    CURAND_RNG_PSEUDO_PHILOX4_32_10 = 161
    assert lib.curandCreateGeneratorHost(ctypes.byref(gen), CURAND_RNG_PSEUDO_PHILOX4_32_10) == 0
    try:
        assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        assert lib.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(4 * first_block)) == 0
        out = (ctypes.c_uint * (4 * nblocks))()
        assert lib.curandGenerate(gen, out, ctypes.c_size_t(4 * nblocks)) == 0
    finally:
        lib.curandDestroyGenerator(gen)
    return np.array(out[:], dtype=np.uint32).reshape(nblocks, 4)


def test_philox_matches_curand_host_generator(orc):
    # An independent Philox4x32-10: cuRAND's host generator, keyed by the 64-bit seed.  Its
    # output stream runs 65536 subsequences side by side: block j of four words is the bijection
    # at counter (n_lo, n_hi, j mod 65536, 0) with n = j div 65536 (observed from its outputs).
    # That pins both key words and counter words 0-2 of the oracle's implementation.
    lib = _curand_host_lib()
    if lib is None:
        pytest.skip("libcurand not found")
    for seed in (0, 1, 0x0123456789ABCDEF, 0xDEADBEEF12345678, 2 ** 64 - 1):
        key = [seed & 0xFFFFFFFF, seed >> 32]
        for j0, n in ((0, 64), (65530, 12), (5 * 65536 + 77, 4), ((1 << 40) + 12345, 3),
                      ((1 << 48) + 7, 3), ((1 << 60) + (1 << 50) + 99, 2)):
            got = _curand_host_philox_blocks(lib, seed, j0, n)
            for q in range(n):
                j = j0 + q
                c = j >> 16
                ref = orc.philox4x32_10([c & 0xFFFFFFFF, c >> 32, j & 0xFFFF, 0], key)
                assert np.array_equal(got[q], ref), (hex(seed), j)