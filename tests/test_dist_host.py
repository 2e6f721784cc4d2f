"""The multi-process path of bench.py on CPU: two gloo ranks (replicas) take
the maximum of their step times and report the whole job's throughput."""
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


def _rank_main(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        ms = bench.max_over_ranks(times[rank], world)
        out[rank] = (ms, bench.job_throughput(1000.0, world, ms))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, times = 2, [12.5, 20.0]
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), times, out), nprocs=world,
                           join=True, start_method="spawn")
        got = dict(out)
    for rank in range(world):
        ms, tput = got[rank]
        assert ms == pytest.approx(20.0)
        assert tput == pytest.approx(1000.0 * world / 0.020)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(100.0, 1, 10.0) == pytest.approx(1e4)
