"""Multi-process host logic of the benchmark, on CPU with the gloo backend
(world size 2): each rank scans its own shard (distinct seeds, same shape),
the timed region is closed by barriers, the reported time is the max over
ranks and the throughput sums the ranks' work."""
import os
import socket

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
