"""Plumbing of the vocab-sharded pass: one process per GPU, each holding a contiguous slice of
the vocabulary of every logit row (as a tensor-parallel LM head leaves them).

A step on each rank is three library calls with two all-gathers of fixed-size per-row records
between them (``include/svd_vocab.h``); in stochastic mode an element-wise max over ranks then
brings the correction / bonus token, written only by the rank whose slice holds it, to every
rank.  Every rank combines the gathered records with the same code, so decisions agree without
any further exchange and no kernel waits for another rank.

``run_emulated`` makes the same calls for all P slices on one device, with device copies in
place of the all-gathers: the single-GPU check of the sharded arithmetic.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import api


def vocab_slices(V: int, P: int, align: int = 8) -> List[Tuple[int, int]]:
    """[(v0, Vl)] of P contiguous slices tiling [0, V).  Slice sizes are multiples of ``align``
    (the kernels' 16-byte fast path) except the last, when V holds at least P such groups;
    otherwise an even split by ids."""
    if V < P or P < 1:
        raise ValueError("need 1 <= P <= V")
    groups, tail = divmod(V, align)
    out = []
    if groups >= P:
        base, extra = divmod(groups, P)
        v0 = 0
        for r in range(P):
            n = (base + (1 if r < extra else 0)) * align
            if r == P - 1:
                n += tail
            out.append((v0, n))
            v0 += n
    else:
        base, extra = divmod(V, P)
        v0 = 0
        for r in range(P):
            n = base + (1 if r < extra else 0)
            out.append((v0, n))
            v0 += n
    return out


def _world(group=None) -> int:
    if not (dist.is_available() and dist.is_initialized()):
        return 1
    return dist.get_world_size(group)


def all_gather_records(recv: torch.Tensor, send: torch.Tensor, group=None) -> None:
    """recv[r * len(send):(r + 1) * len(send)] = send of rank r (rank order of ``group``)."""
    n = send.numel()
    world = _world(group)
    if world == 1:
        recv[:n].copy_(send)
        return
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(recv[:world * n], send, group=group)
    else:
        parts = [torch.empty_like(send) for _ in range(world)]
        dist.all_gather(parts, send, group=group)
        recv[:world * n].copy_(torch.cat(parts))


def combine_sampled(emitted: torch.Tensor, row_info: Optional[torch.Tensor] = None,
                    group=None) -> None:
    """Stochastic mode: the correction / bonus token sits only on its owner (-1 elsewhere), all
    other entries agree, so an element-wise max over ranks completes ``emitted`` (and the
    ``sample_token`` column of ``row_info``) on every rank."""
    if _world(group) == 1:
        return
    dist.all_reduce(emitted, op=dist.ReduceOp.MAX, group=group)
    if row_info is not None:
        col = row_info[..., 3].contiguous()
        dist.all_reduce(col, op=dist.ReduceOp.MAX, group=group)
        row_info[..., 3] = col


def step(shard: api.VocabShard, group=None, stream=None) -> dict:
    """One rank's vocab-sharded verify-and-distill step (every rank of ``group`` calls it)."""
    shard.stats(stream)
    all_gather_records(shard.recv1, shard.send1, group)
    shard.resolve(stream)
    all_gather_records(shard.recv2, shard.send2, group)
    shard.finish(stream)
    if shard.stochastic:
        combine_sampled(shard.emitted, shard.row_info, group)
    return shard.outputs()


def run_emulated(shards: Sequence[api.VocabShard], stream=None) -> None:
    """All ranks' calls on one device, in the order the ranks make them; device copies stand
    in for the all-gathers and an element-wise max for the stochastic combine."""
    def gather(name_send, name_recv):
        sends = [getattr(s, name_send) for s in shards]
        g = torch.cat(sends)
        for s in shards:
            getattr(s, name_recv)[:g.numel()].copy_(g)

    for s in shards:
        s.stats(stream)
    gather("send1", "recv1")
    for s in shards:
        s.resolve(stream)
    gather("send2", "recv2")
    for s in shards:
        s.finish(stream)
    if shards[0].stochastic:
        em = shards[0].emitted.clone()
        for s in shards[1:]:
            em = torch.maximum(em, s.emitted)
        for s in shards:
            s.emitted.copy_(em)
        if shards[0].row_info is not None:
            col = shards[0].row_info[..., 3].clone()
            for s in shards[1:]:
                col = torch.maximum(col, s.row_info[..., 3])
            for s in shards:
                s.row_info[..., 3] = col
