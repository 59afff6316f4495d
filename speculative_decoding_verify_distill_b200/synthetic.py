"""Seeded synthetic inputs shaped like the serving workloads of the AdaFlash pages.

This module holds the input recipe only: random numbers, shapes and scales.  It computes none
of the verify/accept/distill arithmetic, so both the CUDA path (through the tests and the
benchmark) and the CPU oracle can be fed from it without sharing any of the method's code.

Recipe (stated once, used everywhere):
  * one seeded random permutation pi of the vocabulary per workload; per-id bias
    ``-log(pi(v) + 1)`` gives the Zipf-like head/tail of an LLM output distribution;
  * target logits ``T[b,i,v] = 2 * N(0,1) + bias[v]`` drawn in fp32, rounded RNE to bf16;
  * draft logits ``D[b,i,v] = T_fp32[b,i,v] + sigma * N(0,1)`` rounded RNE to bf16, where sigma
    grows with the draft position (later positions are worse drafts) or is drawn per sequence;
  * pooled drafter hidden states ``h = gain * N(0,1)`` and a random length head
    ``W1, w2 ~ N(0, 0.02^2)``, zero biases;
  * stochastic-mode draft tokens are samples of ``softmax(D/tau)`` drawn by the Gumbel-max trick.

Every sequence b draws from its own generator seeded from (workload seed, b), so any subset of
sequences can be regenerated on the host without producing the whole batch.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import math
import os
from typing import Optional, Sequence

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    k: int
    V: int
    kt: int
    H: int
    M: int
    seed: int
    sigma: tuple             # ("pos", a, b): a + b*i   |   ("seq", lo, hi): U(lo, hi) per sequence
    gain: float = 1.0
    mode: int = 0            # 0 greedy, 1 stochastic
    lam: float = 0.5
    clip_c: float = 1.0
    tau: float = 1.0
    philox_seed: int = 0

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads.  Sizes follow the serving settings the pages discuss: concurrency up to
# 128 sequences, blocks of k = 8..16 drafts, Qwen3-class (151936) and Llama-3-class (128256)
# vocabularies.
WORKLOADS = {
    "tiny": Workload("tiny", B=4, k=8, V=1024, kt=8, H=256, M=64, seed=100,
                     sigma=("pos", 0.5, 0.15)),
    "greedy_qwen_b32": Workload("greedy_qwen_b32", B=32, k=16, V=151936, kt=16, H=4096, M=256,
                                seed=101, sigma=("pos", 0.5, 0.15)),
    "ragged_qwen_b128": Workload("ragged_qwen_b128", B=128, k=16, V=151936, kt=16, H=4096, M=256,
                                 seed=102, sigma=("seq", 0.2, 2.0), gain=8.0),
    "stochastic_qwen_b64": Workload("stochastic_qwen_b64", B=64, k=16, V=151936, kt=16, H=4096,
                                    M=256, seed=103, sigma=("pos", 0.5, 0.15), mode=1,
                                    philox_seed=1234),
    "stress_llama_b256": Workload("stress_llama_b256", B=256, k=16, V=128256, kt=16, H=4096,
                                  M=256, seed=104, sigma=("pos", 0.3, 0.2)),
}
# Order of the workloads as listed in the problem statement (tiny first).
WORKLOAD_ORDER = ["tiny", "greedy_qwen_b32", "ragged_qwen_b128", "stochastic_qwen_b64",
                  "stress_llama_b256"]
# The clipping / mixing sweep of the stress workload.
STRESS_SWEEP = [(c, lam) for c in (0.1, 1.0, math.inf) for lam in (0.0, 0.5, 1.0)]


def _gen(seed: int, stream: int, b: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed((seed * 1_000_003 + stream * 7_919 + b + 1) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def vocab_bias(w: Workload) -> torch.Tensor:
    """-log(pi(v) + 1) for a seeded permutation pi of the ids (fp32, [V])."""
    g = _gen(w.seed, 0, -1)
    rank = torch.randperm(w.V, generator=g)
    return -torch.log(rank.to(torch.float64) + 1.0).to(torch.float32)


def sequence_sigmas(w: Workload, b: int) -> list:
    """Draft noise scale per position of sequence b."""
    kind, a, c = w.sigma
    if kind == "seq":
        g = _gen(w.seed, 1, b)
        s = a + (c - a) * torch.rand(1, generator=g, dtype=torch.float64).item()
        return [s] * w.k
    return [a + c * i for i in range(w.k)]


def _one_sequence(w: Workload, b: int, bias: torch.Tensor):
    g = _gen(w.seed, 2, b)
    t32 = 2.0 * torch.randn((w.kt, w.V), generator=g, dtype=torch.float32) + bias
    sig = torch.tensor(sequence_sigmas(w, b), dtype=torch.float32).view(w.k, 1)
    d32 = t32[: w.k] + sig * torch.randn((w.k, w.V), generator=g, dtype=torch.float32)
    return d32.to(torch.bfloat16), t32.to(torch.bfloat16)


def make_logits(w: Workload, seqs: Optional[Sequence[int]] = None, threads: Optional[int] = None,
                pin: bool = False):
    """Draft and target logits for the sequences `seqs` (default: all B).

    Returns (D [n,k,V] bf16, T [n,kt,V] bf16) on the CPU; row b of the output is sequence
    seqs[b] of the workload.
    """
    seqs = list(range(w.B)) if seqs is None else list(seqs)
    n = len(seqs)
    bias = vocab_bias(w)
    D = torch.empty((n, w.k, w.V), dtype=torch.bfloat16, pin_memory=pin)
    T = torch.empty((n, w.kt, w.V), dtype=torch.bfloat16, pin_memory=pin)
    threads = threads or min(32, os.cpu_count() or 1)

    def work(j):
        d, t = _one_sequence(w, seqs[j], bias)
        D[j].copy_(d)
        T[j].copy_(t)

    if n <= 2 or threads == 1:
        for j in range(n):
            work(j)
    else:
        prev = torch.get_num_threads()
        torch.set_num_threads(1)
        try:
            with _cf.ThreadPoolExecutor(max_workers=threads) as ex:
                list(ex.map(work, range(n)))
        finally:
            torch.set_num_threads(prev)
    return D, T


def make_head(w: Workload, B: Optional[int] = None):
    """Length-head inputs: h [B,H] bf16, W1 [M,H] bf16, b1 [M] fp32 (zeros), w2 [M] bf16, b2."""
    B = w.B if B is None else B
    g = _gen(w.seed, 3, -1)
    W1 = (0.02 * torch.randn((w.M, w.H), generator=g)).to(torch.bfloat16)
    w2 = (0.02 * torch.randn((w.M,), generator=g)).to(torch.bfloat16)
    gh = _gen(w.seed, 4, -1)
    h = (w.gain * torch.randn((B, w.H), generator=gh)).to(torch.bfloat16)
    b1 = torch.zeros(w.M, dtype=torch.float32)
    return h, W1, b1, w2, 0.0


def sample_draft_tokens(D: torch.Tensor, tau: float, seed: int, seqs: Optional[Sequence[int]] = None):
    """Draft tokens x[b,i] ~ softmax(D[b,i]/tau) by the Gumbel-max trick (int32 [n,k])."""
    n, k, V = D.shape
    seqs = list(range(n)) if seqs is None else list(seqs)
    out = torch.empty((n, k), dtype=torch.int32)
    for j in range(n):
        g = _gen(seed, 5, seqs[j])
        u = torch.rand((k, V), generator=g, dtype=torch.float64).clamp_min(1e-300)
        gumbel = -torch.log(-torch.log(u))
        out[j] = torch.argmax(D[j].to(torch.float64) / tau + gumbel, dim=-1).to(torch.int32)
    return out


def sample_draft_tokens_batched(D: torch.Tensor, tau: float, seed: int):
    """Same law as sample_draft_tokens, one generator for the whole (small) batch."""
    g = _gen(seed, 7, -1)
    u = torch.rand(D.shape, generator=g, dtype=torch.float64).clamp_min(1e-300)
    gumbel = -torch.log(-torch.log(u))
    return torch.argmax(D.to(torch.float64) / tau + gumbel, dim=-1).to(torch.int32)


def random_bk(B: int, k: int, seed: int) -> torch.Tensor:
    """Verification lengths drawn uniformly from 1..k (for tests that bypass the length head)."""
    g = _gen(seed, 6, -1)
    return torch.randint(1, k + 1, (B,), generator=g, dtype=torch.int32)
