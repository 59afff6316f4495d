"""The vocab-sharded step's host plumbing on CPU: slice tiling, and two or three gloo ranks running
``vocab_parallel.step`` over a fake of the three library calls.  The fake records what each
call saw, so the test checks the order of calls and exchanges, that every rank's records land
at its rank's block of the gathered buffers before the next call reads them, and the
stochastic max-combine of the sampled token."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from speculative_decoding_verify_distill_b200 import vocab_parallel as vp


@pytest.mark.parametrize("V", [1, 7, 64, 1000, 1024, 151936, 128256])
@pytest.mark.parametrize("P", [1, 2, 3, 8])
def test_vocab_slices_tile_the_vocabulary(V, P):
    if V < P:
        with pytest.raises(ValueError):
            vp.vocab_slices(V, P)
        return
    for align in (1, 8):
        sl = vp.vocab_slices(V, P, align)
        assert len(sl) == P
        v = 0
        for r, (v0, n) in enumerate(sl):
            assert v0 == v and n >= 1
            v += n
        assert v == V
        if V // align >= P:
            assert all(n % align == 0 for _, n in sl[:-1])
            sizes = [n for _, n in sl[:-1]]
            assert max(sizes, default=0) - min(sizes, default=0) <= align


class FakeShard:
    """Stands in for api.VocabShard: same buffers and calls, CPU tensors, no arithmetic."""

    def __init__(self, rank, P, n1=12, n2=8, B=3, k=4, stochastic=True):
        self.rank, self.P = rank, P
        self.send1 = torch.zeros(n1, dtype=torch.uint8)
        self.recv1 = torch.zeros(P * n1, dtype=torch.uint8)
        self.send2 = torch.zeros(n2, dtype=torch.uint8)
        self.recv2 = torch.zeros(P * n2, dtype=torch.uint8)
        self.emitted = torch.full((B, k + 1), -1, dtype=torch.int32)
        self.row_info = torch.full((B, k, 8), -1, dtype=torch.int32)
        self.stochastic = stochastic
        self.log = []

    def stats(self, stream=None):
        self.log.append("stats")
        self.send1.fill_(10 + self.rank)

    def resolve(self, stream=None):
        self.log.append(("resolve", self.recv1.clone()))
        self.send2.fill_(20 + self.rank)
        self.emitted[:, 0] = 5                       # identical on every rank

    def finish(self, stream=None):
        self.log.append(("finish", self.recv2.clone()))
        # the sampled token of sequence b lives on rank b % P
        for b in range(self.emitted.shape[0]):
            if b % self.P == self.rank:
                self.emitted[b, 1] = 100 + b
                self.row_info[b, 1, 3] = 100 + b

    def outputs(self):
        return dict(emitted=self.emitted)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        sh = FakeShard(rank, world)
        out = vp.step(sh)
        q.put((rank, sh.log[0], sh.log[1][0], sh.log[1][1].tolist(), sh.log[2][0],
               sh.log[2][1].tolist(), out["emitted"].tolist(), sh.row_info[..., 3].tolist()))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_multi_rank_step_gloo(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    emitted = []
    for rank, c0, c1, recv1, c2, recv2, em, ri in res:
        assert (c0, c1, c2) == ("stats", "resolve", "finish")
        assert recv1 == sum(([10 + r] * 12 for r in range(world)), [])   # rank r at block r
        assert recv2 == sum(([20 + r] * 8 for r in range(world)), [])
        emitted.append(em)
        for b in range(3):
            assert em[b][0] == 5 and em[b][1] == 100 + b   # max-combined sampled token
            assert ri[b][1] == 100 + b
    assert all(e == emitted[0] for e in emitted)


def test_single_process_step_is_local():
    sh = FakeShard(0, 1)
    vp.step(sh)
    assert sh.log[1][1].tolist() == [10] * 12 and sh.log[2][1].tolist() == [20] * 8
    assert [sh.emitted[b, 1].item() for b in range(3)] == [100, 101, 102]
