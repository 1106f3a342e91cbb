"""The N > 1 path of bench.py: independent replicas, one per rank, timed as
the slowest rank (max over ranks), aggregate = all ranks' units / that time.
Runs as two gloo ranks on CPU."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        my_ms = [30.0, 45.0][rank]  # rank 1 is the slow one
        t, rate = bench.aggregate_ranks(my_ms, units_per_rank_step=1000, steps=3, world=world,
                                        reduce_max=bench.dist_max(dist, "cpu"))
        out[rank] = (t, rate)
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_take_the_slowest_rank():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        t, rate = out[r]
        assert t == 45.0                              # max over ranks
        assert rate == pytest.approx(2 * 1000 * 3 / 0.045)  # every rank's units / slowest time


def test_single_rank_is_identity():
    t, rate = bench.aggregate_ranks(20.0, 500, 4, 1, None)
    assert t == 20.0 and rate == pytest.approx(500 * 4 / 0.02)
