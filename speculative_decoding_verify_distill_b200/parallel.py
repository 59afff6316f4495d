"""Data-parallel plumbing for the verify-and-distill pass (one process per GPU).

Sequences are independent: b_k, acceptance, loss rows and gradient rows never cross sequences,
so a batch shards on the sequence axis with no exchange in the data path.  Each rank runs its
own batch of B sequences (weak scaling).  The only collectives are host-level reductions of the
per-step scalars: the device time (max over ranks), the token counts and the loss (sums).
"""
from __future__ import annotations

import dataclasses
import os
from typing import Optional

import torch
import torch.distributed as dist


@dataclasses.dataclass
class RankInfo:
    rank: int
    world: int
    local_rank: int


def init_from_env(backend: str = "nccl", timeout_s: int = 300) -> RankInfo:
    """Joins the process group described by RANK / WORLD_SIZE / LOCAL_RANK (torchrun)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    return RankInfo(rank, world, local)


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s batch: rank 0 keeps the workload's own seed."""
    return base_seed + 7919 * rank


def shard_range(B: int, rank: int, world: int):
    """Contiguous [lo, hi) slice of B sequences for strong-scaling splits of one batch."""
    base, extra = divmod(B, world)
    lo = rank * base + min(rank, extra)
    hi = lo + base + (1 if rank < extra else 0)
    return lo, hi


def reduce_metrics(ms: float, verified: float, accepted: float, emitted: float, loss: float,
                   device: Optional[torch.device] = None) -> dict:
    """Max of the step time, sums of the token counts and losses over all ranks."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return dict(ms=ms, verified=verified, accepted=accepted, emitted=emitted, loss=loss)
    dev = device or torch.device("cpu")
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    s = torch.tensor([verified, accepted, emitted, loss], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(s, op=dist.ReduceOp.SUM)
    return dict(ms=float(t[0]), verified=float(s[0]), accepted=float(s[1]), emitted=float(s[2]),
                loss=float(s[3]))
