"""Multi-rank plumbing of the bench on CPU: world size 2 over gloo.

The decode step has no cross-GPU data exchange (ranks are independent
replicas); what runs across ranks is the sharding of sequences, the barrier
around the timed region and the max/sum over ranks of the measurements.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

from rank_kv_cache_palu_b200 import dist as D


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, _ = D.init("gloo", timeout_s=30)
    lo, hi = D.shard(37, r, w)
    D.barrier()
    mx = D.max_over_ranks(float(10 + r))
    tot = D.sum_over_ranks(float(hi - lo))
    q.put((r, lo, hi, mx, tot))
    D.finalize()


def test_two_rank_shard_barrier_and_reductions():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=60) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, lo0, hi0, mx0, tot0), (r1, lo1, hi1, mx1, tot1) = res
    assert (lo0, hi1) == (0, 37) and hi0 == lo1            # a partition of the 37 sequences
    assert mx0 == mx1 == 11.0
    assert tot0 == tot1 == 37.0


@pytest.mark.parametrize("n,world", [(16, 1), (16, 3), (5, 8), (0, 2)])
def test_shard_partitions(n, world):
    seen = []
    for r in range(world):
        lo, hi = D.shard(n, r, world)
        assert 0 <= lo <= hi <= n
        seen.extend(range(lo, hi))
    assert seen == list(range(n))
