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


def test_reference_arm_prints_one_contract_line():
    # the reference arm (the CPU oracle on a bounded sample) runs without a GPU: one JSON line
    # with the arm's own metric, unit and config, a cpu_baseline describing the run and an e2e
    # entry that moves no bytes
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 3
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["config"]["workload"] == "dit_mlp_pair_m4096_h3072_f12288"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_oracle_thread_count(monkeypatch):
    # the cores a CPU-baseline line states are the oracle's OpenMP threads
    import os
    import bench
    monkeypatch.setenv("OMP_NUM_THREADS", "3")
    assert bench.oracle_threads() == 3
    monkeypatch.delenv("OMP_NUM_THREADS")
    assert bench.oracle_threads() == len(os.sched_getaffinity(0))
