"""Comparison helpers shared by the GPU parity tests (test infrastructure).

Tolerances (stated once):
  * integers (argmax, b_k, accepted lengths, emitted tokens, sampled tokens): bit-exact, except
    the counted near-ties of the decision readings below;
  * losses, lse and fp32 gradients: |gpu - oracle| <= max(ATOL, RTOL * |oracle|) with
    RTOL = 1e-3, ATOL = 1e-5 (fp32 accumulation against the fp64 oracle);
  * bf16 gradients: within one bf16 ulp of RNE(oracle), or within ATOL of the oracle;
  * clip decisions: an entry whose d_v = q_v s_v lies within TIE_CLIP * q_v (1 + |s_v|) of c
    (oracle values; the fp32 error of d_v is below a third of that) may be clipped on one side
    and not on the other.  Such "band" entries are counted, left out of the element-wise
    gradient comparison, and every other entry of the row is compared with the tolerance above
    widened by the most their flips can move the row's sums: (scale/tau)(1 - lambda) q_u dS for
    the gradient, (1 - lambda) dK for the row loss (dS, dK from oracle.clip_band).  Band
    entries must stay under 1% of each row;
  * stochastic accept decisions: identical unless |u - p/q| < 1e-6 (oracle values);
  * sampled tokens: identical unless the oracle's sample point lies within 1e-6 * R of a
    running-sum boundary;
  * b_k: identical unless gamma * bhat * k lies within 1e-4 of an integer (oracle value).
"""
from __future__ import annotations

import math

import numpy as np
import torch

RTOL, ATOL = 1e-3, 1e-5
TIE_U = 1e-6
TIE_SAMPLE = 1e-6
TIE_BK = 1e-4
TIE_CLIP = 2e-5
BAND_MAX_FRAC = 0.01


def close_mask(gpu, ref, rtol=RTOL, atol=ATOL):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    return np.abs(gpu - ref) <= np.maximum(atol, rtol * np.abs(ref))


def assert_close(gpu, ref, what, rtol=RTOL, atol=ATOL, mask=None, extra=None):
    """|gpu - ref| <= max(atol, rtol |ref|) (+ extra, a per-element widening) where mask is set."""
    ok = close_mask(gpu, ref, rtol, atol)
    if extra is not None:
        d = np.abs(np.asarray(gpu, np.float64) - np.asarray(ref, np.float64))
        ok = ok | (d <= np.maximum(atol, rtol * np.abs(np.asarray(ref, np.float64))) + extra)
    if mask is not None:
        ok = ok | ~mask
    if not ok.all():
        g = np.asarray(gpu, np.float64)
        r = np.asarray(ref, np.float64)
        bad = np.argwhere(~ok)
        i = tuple(bad[0])
        raise AssertionError("%s: %d/%d outside tolerance; first at %s gpu=%r oracle=%r"
                             % (what, (~ok).sum(), ok.size, i, g[i], r[i]))


def bf16_round(x: np.ndarray) -> np.ndarray:
    """RNE of float64 values to bf16, returned as float64 (via fp32, the kernel's output path)."""
    t = torch.from_numpy(np.asarray(x, np.float64)).to(torch.float32).to(torch.bfloat16)
    return t.to(torch.float64).numpy()


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(np.asarray(x, np.float64))
    ax = np.where(ax < 2.0 ** -126, 2.0 ** -126, ax)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def assert_bf16_grad(gpu_bf16: torch.Tensor, ref: np.ndarray, what: str, mask=None, extra=None):
    g = gpu_bf16.detach().to(torch.float64).cpu().numpy()
    r = np.asarray(ref, np.float64)
    rr = bf16_round(r)
    e = 0.0 if extra is None else extra
    ok = (np.abs(g - rr) <= bf16_ulp(rr) + e) | (np.abs(g - r) <= ATOL + e)
    if mask is not None:
        ok = ok | ~mask
    if not ok.all():
        bad = np.argwhere(~ok)
        i = tuple(bad[0])
        raise AssertionError("%s: %d/%d bf16 values off by more than 1 ulp; first at %s gpu=%r "
                             "oracle=%r" % (what, (~ok).sum(), ok.size, i, g[i], r[i]))


def bk_near_integer(bhat: np.ndarray, k: int, gamma: float = 1.0) -> np.ndarray:
    x = gamma * np.asarray(bhat, np.float64) * k
    return np.abs(x - np.round(x)) < TIE_BK


def clip_band(D, T, bk, c: float, tau: float, want_mask: bool = True) -> dict:
    """Band entries of the verified rows (see the module docstring) from the oracle, with the
    per-row fraction checked against BAND_MAX_FRAC."""
    import oracle
    cb = oracle.clip_band(D, T, bk, c, tau, TIE_CLIP, want_mask=want_mask)
    V = D.shape[2]
    worst = cb["n_band"].max() if cb["n_band"].size else 0
    assert worst <= max(1.0, BAND_MAX_FRAC * V), ("clip band too wide for an element-wise comparison",
                                        int(worst), V)
    return cb


def softmax_rows(X, tau: float) -> np.ndarray:
    """q = softmax(X / tau) of bf16 rows in fp64 (the tolerance widening only)."""
    return torch.softmax(X.double() / tau, -1).numpy()
