"""Host logic of the multi-GPU bench path, as two gloo ranks on the CPU:
each rank gets its own shard (weak scaling, no data-path collective) and the
reported time is the max over ranks."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        plan = bench.shard_for_rank(rank, world)
        mine = 10.0 + rank * 5.0
        got = bench.max_over_ranks(mine, dist)
        seeds = [None] * world
        dist.all_gather_object(seeds, plan["seed"])
        out[rank] = (got, seeds)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    # spawn, not fork: earlier tests may have started OpenMP threads
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        got, seeds = res[r]
        assert got == 15.0                       # the max over ranks
        assert len(set(seeds)) == world          # distinct shards


def test_shard_plan():
    plans = [bench.shard_for_rank(r, 4) for r in range(4)]
    assert len({p["seed"] for p in plans}) == 4
    with pytest.raises(ValueError):
        bench.shard_for_rank(4, 4)
    assert bench.max_over_ranks(3.5) == 3.5
