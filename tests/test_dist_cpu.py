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


def shard_worker(rank, world, port, q, bounds):
    """One rank of a sequence-sharded forward on the CPU: the slice summaries
    come from the oracle, the exchange is the product's all-gather (gloo),
    the prefix and the slice's solve follow the definitions."""
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import numpy as np
    import torch
    import torch.distributed as dist
    import oracle
    from test_oracle_pins import rand_inputs
    from test_sequence_layer_b200 import sharded
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        x = rand_inputs(np.random.default_rng(3), 2, 2, bounds[-1], 4, 4)
        t0, t1 = bounds[rank], bounds[rank + 1]
        qs, ks, vs = (a[:, :, t0:t1] for a in x[:3])
        gs, bs = x[3][:, :, t0:t1], x[4][:, :, t0:t1]
        _, _, Hd, Gd = oracle.forward_cg(qs, ks, vs, gs, bs, x[5], 6)          # slice from a zero state
        dec = np.prod(gs, axis=-1)
        H_all, G_all, d_all = sharded.gather_slice_summaries(torch.from_numpy(Hd), torch.from_numpy(Gd),
                                                             torch.from_numpy(dec))
        S_H, S_G = np.zeros_like(Hd), np.zeros_like(Gd)
        for s in range(rank):                          # S_{s+1} = D_s S_s + Delta_s
            D = d_all[s].numpy()[..., None, None]
            S_H, S_G = D * S_H + H_all[s].numpy(), D * S_G + G_all[s].numpy()
        out, _, _, _ = oracle.forward_cg(qs, ks, vs, gs, bs, x[5], 6, H0=S_H, G0=S_G)
        dist.barrier()
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("bounds", [(0, 9, 20), (0, 5, 6, 17)])
def test_sequence_sharded_forward_equals_whole(bounds):
    """Ranks own consecutive slices (uneven, one of length 1); the outputs,
    put together in rank order, equal the unsharded forward."""
    import sys
    import numpy as np
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from test_oracle_pins import rand_inputs
    world = len(bounds) - 1
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=shard_worker, args=(r, world, port, q, bounds)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = rand_inputs(np.random.default_rng(3), 2, 2, bounds[-1], 4, 4)
    whole, _, _, _ = oracle.forward_cg(*x, 6)
    got = np.concatenate([res[r] for r in range(world)], axis=2)
    np.testing.assert_allclose(got, whole, rtol=1e-10, atol=1e-12)
