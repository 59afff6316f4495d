"""Comparison helpers shared by the GPU parity tests (test infrastructure).

Tolerances (stated once):
  * integers (argmax, b_k, accepted lengths, emitted tokens, sampled tokens): bit-exact, except
    the counted near-ties of the decision readings below;
  * losses, lse and fp32 gradients: |gpu - oracle| <= max(ATOL, RTOL * |oracle|) with
    RTOL = 1e-3, ATOL = 1e-5 (fp32 accumulation against the fp64 oracle);
  * bf16 gradients: within one bf16 ulp of RNE(oracle), or within ATOL of the oracle;
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


def close_mask(gpu, ref, rtol=RTOL, atol=ATOL):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    return np.abs(gpu - ref) <= np.maximum(atol, rtol * np.abs(ref))


def assert_close(gpu, ref, what, rtol=RTOL, atol=ATOL, mask=None):
    ok = close_mask(gpu, ref, rtol, atol)
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


def assert_bf16_grad(gpu_bf16: torch.Tensor, ref: np.ndarray, what: str, mask=None):
    g = gpu_bf16.detach().to(torch.float64).cpu().numpy()
    r = np.asarray(ref, np.float64)
    rr = bf16_round(r)
    ok = (np.abs(g - rr) <= bf16_ulp(rr)) | (np.abs(g - r) <= ATOL)
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


def near_clip_rows(D, T, bk, c: float, tau: float, seqs=None) -> np.ndarray:
    """[B,k] mask of verified rows that hold an entry with |d_v - c| < 1e-5 * max(1, c): the
    clip decision of such an entry is not fixed by fp32 arithmetic (counted, not compared)."""
    B, k, V = D.shape
    out = np.zeros((B, k), bool)
    if not math.isfinite(c):
        return out
    for b in range(B):
        n = int(bk[b])
        for i in range(n):
            lq = torch.log_softmax(D[b, i].double() / tau, -1)
            lp = torch.log_softmax(T[b, i].double() / tau, -1)
            d = lq.exp() * (lq - lp)
            out[b, i] = bool(((d - c).abs() < 1e-5 * max(1.0, c)).any())
    return out
