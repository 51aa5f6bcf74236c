"""The bench's multi-rank bookkeeping on CPU: two gloo ranks (one process each, as one process
per GPU runs on the box), each with its own step time; every rank must see the slowest time,
and the whole-job throughput counts both ranks' work over that time (weak scaling)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(times[rank], dist, torch.device("cpu"))
        out[rank] = ms
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    times = [0.040, 0.052]
    out = mp.Manager().dict()
    mp.start_processes(_rank_main, args=(world, port, times, out), nprocs=world,
                       start_method="spawn", join=True)
    assert out[0] == out[1] == max(times)


def test_job_throughput_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    flops = 2.0 * 4096 * 3072 * 3072
    one = bench.job_tflops(1, 0.044, flops)
    assert bench.job_tflops(2, 0.044, flops) == pytest.approx(2 * one)
    assert one == pytest.approx(flops / 0.044e-3 / 1e12)
    assert bench.max_over_ranks(0.044, None, torch.device("cpu")) == 0.044
