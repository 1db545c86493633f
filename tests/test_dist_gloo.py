"""The data-parallel plumbing on CPU: two gloo ranks in child processes.

Sequences are independent, so ranks share no data; the host logic under test
is the sharding of units over ranks, per-rank seeds, and the max/sum over
ranks that the benchmark's timing and throughput use."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    from mla_latent_kv_19_b200 import dist
    r, _, w = dist.init("gloo", timeout_s=60)
    assert (r, w) == (rank, world)
    begin, end = dist.shard(13, r, w)
    slowest = dist.max_over_ranks(1.5 + r)          # "step times" 1.5 and 2.5 ms
    total = dist.sum_over_ranks(end - begin)
    dist.barrier()
    q.put((r, begin, end, slowest, total, dist.rank_seed(1, r)))
    dist.finish()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    (r0, b0, e0, s0, t0, seed0), (r1, b1, e1, s1, t1, seed1) = res
    assert (b0, e0, b1, e1) == (0, 7, 7, 13)      # contiguous, sizes differ by at most one
    assert s0 == s1 == 2.5                         # every rank sees the slowest rank's time
    assert t0 == t1 == 13                          # all units accounted for once
    assert seed0 != seed1


@pytest.mark.parametrize("n,world", [(32, 1), (32, 3), (5, 8), (0, 2)])
def test_shard_covers_every_unit_once(n, world):
    from mla_latent_kv_19_b200 import dist
    seen = []
    for r in range(world):
        b, e = dist.shard(n, r, world)
        assert 0 <= e - b <= n // world + 1
        seen.extend(range(b, e))
    assert seen == list(range(n))
