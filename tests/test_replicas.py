"""Host logic of the multi-GPU bench (replicas only: no data-path collective)
run as two gloo ranks on the CPU: the job time is the slowest rank's time and
the rate counts the units of every replica."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        ms = bench.max_over_ranks(times[rank], world, "cpu")
        out[rank] = (ms, bench.replica_rate(1000, ms, world))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    world, port = 2, _free_port()
    times = [12.5, 20.0]
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank, args=(world, port, times, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        ms, rate = res[r]
        assert ms == pytest.approx(20.0)
        assert rate == pytest.approx(2 * 1000 / 0.020)


def test_single_rank_is_unchanged():
    import bench
    assert bench.max_over_ranks(7.0, 1, "cpu") == 7.0
    assert bench.replica_rate(500, 250.0, 1) == pytest.approx(2000.0)
