"""The benchmark's multi-rank host logic on CPU: two gloo ranks (one process
each, rendezvous on 127.0.0.1). The slowest rank's time sets the clock and
the whole-job rate counts every rank's units (weak scaling)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def worker(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = [3.0, 5.0, 4.0, 1.0][rank]                     # per-rank device time
        slowest = bench.max_over_ranks(ms, world, "cpu")
        rate = bench.whole_job_rate(1_000_000, world, slowest)
        dist.barrier()
        q.put((rank, slowest, rate))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_max_over_ranks_and_weak_scaling(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = max([3.0, 5.0, 4.0, 1.0][:world])
    for _, slowest, rate in res:
        assert slowest == want
        assert rate == pytest.approx(world * 1_000_000 / (want / 1e3))


def test_single_rank_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5
    assert bench.whole_job_rate(100, 1, 1000.0) == pytest.approx(100.0)
