"""Multi-process host logic of bench.py with two gloo ranks on CPU: each rank
draws its own batch, the job's time is the slowest rank's, and the whole-job
throughput counts every rank's units (weak scaling, no data exchange)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 1.0 + rank  # rank 1 is the slow one
        t = bench.max_over_ranks(ms, dist)
        value, tmax = bench.aggregate([t] * world, 100.0)
        q.put((rank, t, value, tmax, bench.shard_seed(0, rank)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_gloo_max_over_ranks_and_weak_aggregate(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, value, tmax, seed in res:
        assert t == 2.0 and tmax == 2.0
        assert abs(value - world * 100.0 / 2e-3) < 1e-6
    assert len({r[4] for r in res}) == world  # each rank its own batch


def test_single_rank_needs_no_collective():
    import bench

    assert bench.max_over_ranks(3.5, None) == 3.5
    v, t = bench.aggregate([2.0], 10.0)
    assert t == 2.0 and abs(v - 5000.0) < 1e-9
