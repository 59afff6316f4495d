"""The N > 1 host path on CPU: two gloo ranks exchange the per-step scalars exactly as the
benchmark's NCCL ranks do (max of the device time, sums of the counts), and the sharding
helpers partition a batch without overlap."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from speculative_decoding_verify_distill_b200 import parallel


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    info = parallel.init_from_env("gloo", timeout_s=60)
    try:
        r = parallel.reduce_metrics(ms=1.0 + rank, verified=100.0 * (rank + 1), accepted=10.0,
                                    emitted=11.0 + rank, loss=0.5)
        lo, hi = parallel.shard_range(130, info.rank, info.world)
        q.put((info.rank, r, (lo, hi), parallel.rank_seed(102, info.rank)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_rank_reduction_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, r, rng, seed in res:
        assert r["ms"] == 2.0                       # max over ranks
        assert r["verified"] == 300.0               # sums over ranks
        assert r["accepted"] == 20.0 and r["emitted"] == 23.0 and r["loss"] == 1.0
    assert res[0][2] == (0, 65) and res[1][2] == (65, 130)
    assert res[0][3] == 102 and res[1][3] != 102


def test_shard_range_partitions():
    for B in (1, 7, 128, 129):
        for world in (1, 2, 3, 8):
            cover = []
            for r in range(world):
                lo, hi = parallel.shard_range(B, r, world)
                cover.extend(range(lo, hi))
            assert cover == list(range(B))


def test_single_process_reduction_is_identity():
    r = parallel.reduce_metrics(3.0, 5.0, 2.0, 4.0, 1.5)
    assert r == dict(ms=3.0, verified=5.0, accepted=2.0, emitted=4.0, loss=1.5)
