"""Multi-process host logic on CPU with the gloo backend.

- The benchmark (world size 2): each rank scans its own shard (distinct
  seeds, same shape), the timed region is closed by barriers, the reported
  time is the max over ranks and the throughput sums the ranks' work.
- The time-sharded scan (world sizes 2 and 3, ragged and empty slices): the
  exchange of slice summaries and the order they are applied in.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        assert (r, w, lr) == (rank, world, rank)
        cpu = torch.device("cpu")
        bench.barrier(world, cpu)
        # rank-dependent "elapsed" times: the job is as slow as its slowest rank
        t = bench.reduce_max(1.0 + rank, world, cpu)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.shard_seed(17, rank))
        agg = bench.aggregate(bytes_per_step=1000, elems_per_step=10, steps=4, max_seconds=t, world=world)
        q.put((rank, t, seeds, agg))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, seeds, agg in res:
        assert t == 2.0                                  # max over ranks
        assert len(set(seeds)) == world                  # every rank its own shard
        assert agg["gbs"] == pytest.approx(2 * 1000 * 4 / 2.0 / 1e9)
        assert agg["ms_per_step"] == pytest.approx(500.0)



def test_single_rank_is_identity():
    assert bench.reduce_max(3.5, 1, torch.device("cpu")) == 3.5
    agg = bench.aggregate(12, 3, 2, 1.0, 1)
    assert agg["gbs"] == pytest.approx(24e-9)


# ------------------------------------------------ time axis split over ranks
# The orchestration of scan_gated_rnns_b200.sharded.time_sharded_scan on CPU
# ranks: the per-rank device steps are replaced by the fp64 oracle (summaries
# from two scans of the slice), so what runs is the exchange itself -- which
# slice each rank holds, the all-gather order, the order the earlier ranks'
# summaries are applied in, and that only the first slice starts from the
# sequence's initial state.

class _OracleOps:
    @staticmethod
    def summary(op, p, q):
        import oracle
        B, T, D = p.shape
        if op == "mingru":
            h_zero = oracle.mingru_linear(p, q, np.zeros((B, D)))[:, -1] if T else np.zeros((B, D))
            h_one = oracle.mingru_linear(p, q, np.ones((B, D)))[:, -1] if T else np.ones((B, D))
            pair = np.stack([h_one - h_zero, h_zero], -1)            # h_end = A h + B
        else:
            hi = oracle.minmax(p, q, np.full((B, D), np.inf))[:, -1] if T else np.full((B, D), np.inf)
            lo = oracle.minmax(p, q, np.full((B, D), -np.inf))[:, -1] if T else np.full((B, D), -np.inf)
            pair = np.stack([hi, lo], -1)                              # x_end = max(min(x, U), L)
        return torch.from_numpy(pair)

    @staticmethod
    def combine(op, pairs, rank, init, dtype):
        B, D = pairs.shape[1:3]
        x = init.double().numpy().copy() if init is not None else np.zeros((B, D))
        for r in range(rank):
            a, b = pairs[r, ..., 0].numpy(), pairs[r, ..., 1].numpy()
            x = a * x + b if _OracleOps.op == "mingru" else np.maximum(np.minimum(x, a), b)
        return torch.from_numpy(x)

    @staticmethod
    def scan(op, p, q, init):
        import oracle
        fn = oracle.mingru_linear if op == "mingru" else oracle.minmax
        return torch.from_numpy(fn(p, q, init))


def _sharded_worker(rank, world, port, op, bounds, q):
    import numpy as np  # noqa: F811  (spawned process)
    from scan_gated_rnns_b200.sharded import time_sharded_scan
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(5)
        B, T, D = 2, bounds[-1], 6
        p = torch.randn(B, T, D, generator=g, dtype=torch.float64)
        s = torch.randn(B, T, D, generator=g, dtype=torch.float64)
        init = torch.rand(B, D, generator=g, dtype=torch.float64) + 0.1
        _OracleOps.op = op
        t0, t1 = bounds[rank], bounds[rank + 1]
        out = time_sharded_scan(op, p[:, t0:t1].contiguous(), s[:, t0:t1].contiguous(), init,
                                ops=_OracleOps)
        q.put((rank, out.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("op", ["mingru", "minmax"])
@pytest.mark.parametrize("bounds", [(0, 37, 80), (0, 0, 25, 60), (0, 50, 51, 120)])
def test_time_sharded_scan_matches_one_sequence(op, bounds):
    import oracle
    world = len(bounds) - 1
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_worker, args=(r, world, port, op, bounds, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    g = torch.Generator().manual_seed(5)
    B, T, D = 2, bounds[-1], 6
    p = torch.randn(B, T, D, generator=g, dtype=torch.float64)
    s = torch.randn(B, T, D, generator=g, dtype=torch.float64)
    init = torch.rand(B, D, generator=g, dtype=torch.float64) + 0.1
    full = (oracle.mingru_linear if op == "mingru" else oracle.minmax)(p, s, init)
    got = np.concatenate([res[r] for r in range(world)], axis=1)
    if op == "mingru":
        np.testing.assert_allclose(got, full, rtol=1e-12)
    else:
        np.testing.assert_array_equal(got, full)
