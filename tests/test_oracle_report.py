"""Pins of the oracle's speedup reporter (Pith review page, Referee Report minor comment 1:
E[tau] = (1 - A^(k+1)) / (1 - A) and eta = E[tau] / (rho*k + 1))."""
import math

import numpy as np
import pytest


def test_hand_counted_case(orc):
    # three sequences, k = 4: accepted lengths, verified rows, emitted tokens
    a, n, e = [2, 4, 0], [4, 4, 2], [3, 4, 1]
    out = orc.speedup_report(a, n, e, 4, 0.1)
    # decisions taken: 3 (2 accepted + 1 rejected), 4 (all accepted), 1 (rejected at once)
    acc = 6 / 8
    model = (1 - acc ** 5) / (1 - acc)
    assert out[0] == pytest.approx(8 / 3, rel=1e-15)
    assert out[1] == pytest.approx(0.75, rel=1e-15)
    assert out[2] == pytest.approx(3.05078125, rel=1e-15)
    assert out[2] == pytest.approx(model, rel=1e-15)
    assert out[3] == pytest.approx(3.05078125 / 1.4, rel=1e-15)
    assert out[4] == pytest.approx((8 / 3) / 1.4, rel=1e-15)
    assert out[5] == pytest.approx(10 / 3) and out[6] == pytest.approx(2.0) and out[7] == 3
    # per position: (accepted, reached-and-verified) = (2,3), (2,2), (1,2), (1,1)
    np.testing.assert_allclose(out[8:], [2 / 3, 1.0, 0.5, 1.0], rtol=1e-15)


def test_limits(orc):
    k = 6
    full = orc.speedup_report([k] * 5, [k] * 5, [k + 1] * 5, k, 0.0)
    assert full[1] == 1.0 and full[2] == k + 1 and full[0] == k + 1
    assert (full[8:] == 1.0).all()
    none = orc.speedup_report([0] * 5, [k] * 5, [1] * 5, k, 0.0)
    assert none[1] == 0.0 and none[2] == 1.0
    assert none[8] == 0.0 and np.isnan(none[9:]).all()   # nobody reached position 1


def test_geometric_acceptance_recovers_closed_form(orc):
    # i.i.d. acceptance at rate A, all k verified and a bonus row (kt = k + 1): e = a + 1
    rng = np.random.default_rng(7)
    A, k, B = 0.7, 8, 200000
    accepted = rng.random((B, k)) < A
    a = np.where(accepted.all(1), k, np.argmin(accepted, axis=1)).astype(np.int32)
    out = orc.speedup_report(a, np.full(B, k, np.int32), a + 1, k, 0.05)
    sigma = math.sqrt(A * (1 - A) / (B * 3))
    assert abs(out[1] - A) < 5 * sigma
    closed = (1 - A ** (k + 1)) / (1 - A)
    assert out[0] == pytest.approx(closed, rel=5e-3)
    assert out[2] == pytest.approx(closed, rel=5e-3)
    np.testing.assert_allclose(out[8:], A, atol=0.01)
    assert out[3] == pytest.approx(out[2] / (0.05 * k + 1), rel=1e-15)


def test_rejects_bad_arguments(orc):
    with pytest.raises(ValueError):
        orc.speedup_report([], [], [], 4, 0.0)
