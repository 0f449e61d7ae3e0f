"""CPU: the multi-process replica path of bench.py (one rank per GPU, no
data-path collective) -- the job time is the largest rank time and the
job rate counts every rank's units.  Two gloo ranks on 127.0.0.1."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, times, out):
    sys.path.insert(0, ROOT)
    import datetime
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = bench.max_over_ranks(times[rank], dist, "cpu")
        out[rank] = (ms, bench.job_rate(1000, world, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_max_time_and_job_rate():
    world = 2
    times = [12.5, 20.0]        # ms of each rank's timed region
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_rank, args=(world, port, times, out), nprocs=world,
                       join=True, start_method="spawn")
    for r in range(world):
        ms, rate = out[r]
        assert ms == max(times)
        assert rate == pytest.approx(1000 * world / (max(times) / 1e3))


def test_single_process_is_a_no_op():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, None, "cpu") == 7.0
    assert bench.job_rate(300, 1, 1000.0) == pytest.approx(300.0)
