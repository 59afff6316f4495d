"""svd_speedup_report against the oracle's reporter (Pith review page, Referee Report minor
comment 1: E[tau] = (1 - Acc^(k+1)) / (1 - Acc), eta = E[tau] / (rho*k + 1))."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verify_distill_b200 import api
from speculative_decoding_verify_distill_b200 import synthetic as syn

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from speculative_decoding_verify_distill_b200 import build
    build.build()
    oracle.build()


def _compare(a, n, e, k, rho):
    dev = "cuda"
    got = api.svd_speedup_report(torch.from_numpy(a).to(dev), torch.from_numpy(n).to(dev),
                                 torch.from_numpy(e).to(dev), k, rho)
    torch.cuda.synchronize()
    got = got.cpu().numpy()
    ref = oracle.speedup_report(a, n, e, k, rho)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_allclose(got[ok], ref[ok], rtol=1e-12, atol=0)
    return got


@pytest.mark.parametrize("B,k", [(1, 4), (37, 8), (1000, 16), (4099, 32)])
def test_random_outcomes(B, k):
    rng = np.random.default_rng(B * 100 + k)
    n = rng.integers(1, k + 1, B).astype(np.int32)
    a = np.minimum(rng.geometric(0.25, B) - 1, n).astype(np.int32)
    e = (a + (rng.random(B) < 0.8)).astype(np.int32)
    _compare(a, n, e, k, 0.05)


def test_all_accepted_and_all_rejected():
    k = 16
    full = _compare(np.full(64, k, np.int32), np.full(64, k, np.int32), np.full(64, k, np.int32), k, 0.0)
    assert full[1] == 1.0 and full[2] == k + 1
    _compare(np.zeros(64, np.int32), np.full(64, k, np.int32), np.ones(64, np.int32), k, 0.0)


def test_report_of_a_fused_step():
    w = syn.WORKLOADS["greedy_qwen_b32"]
    D, T = syn.make_logits(w)
    h, W1, b1, w2, b2 = syn.make_head(w)
    vd = api.VerifyDistill(D.cuda(), T.cuda(), head=(h.cuda(), W1.cuda(), b1.cuda(), w2.cuda(), b2),
                           lam=w.lam, clip_c=w.clip_c)
    vd()
    rep = api.svd_speedup_report(vd.accept_len, vd.bk, vd.n_emitted, w.k, 0.1)
    torch.cuda.synchronize()
    ref = oracle.speedup_report(vd.accept_len.cpu().numpy(), vd.bk.cpu().numpy(),
                                vd.n_emitted.cpu().numpy(), w.k, 0.1)
    got = rep.cpu().numpy()
    ok = ~np.isnan(ref)
    np.testing.assert_allclose(got[ok], ref[ok], rtol=1e-12)
    d = api.report_dict(rep)
    assert 1.0 <= d["tau_measured"] <= w.k + 1 and 0.0 <= d["acc"] <= 1.0


def test_bad_arguments():
    L = api.lib()
    x = torch.zeros(4, dtype=torch.int32, device="cuda")
    out = torch.zeros(40, dtype=torch.float64, device="cuda")
    P = api._ptr
    assert L.svd_speedup_report(P(x), P(x), P(x), 4, 0, 0.0, P(out), None) == 1
    assert L.svd_speedup_report(P(x), P(x), P(x), 4, 33, 0.0, P(out), None) == 1
    assert L.svd_speedup_report(P(x), P(x), P(x), 0, 4, 0.0, P(out), None) == 1
    assert L.svd_speedup_report(P(x), P(x), P(x), 4, 4, -1.0, P(out), None) == 1
    assert L.svd_speedup_report(P(x), P(x), P(x), 4, 4, float("nan"), P(out), None) == 1
