"""The N > 1 host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

Each rank runs the whole layer on its own batch (weak scaling, no data-path collective), so
the only cross-rank step is the max of the ranks' device times; the whole-job value is
world x one step's FLOPs over that max.  The reference arm runs on rank 0 alone; other ranks
print nothing and exit 0."""
import json
import os
import socket
import subprocess
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
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        ms = bench.reduce_max(times[rank], dist, torch.device("cpu"))
        out[rank] = (ms, bench.job_tflops(world, ms))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value():
    world, port = 2, _free_port()
    times = [2.5, 3.25]   # ms per step on rank 0 and rank 1
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, times, out), nprocs=world, start_method="spawn", join=True)
    sys.path.insert(0, ROOT)
    import bench
    for r in range(world):
        ms, val = out[r]
        assert ms == max(times)
        assert val == pytest.approx(world * bench.FLOP_STEP / (max(times) * 1e-3) / 1e12)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(1.75, None, torch.device("cpu")) == 1.75
    assert bench.job_tflops(1, 2.0) == pytest.approx(bench.FLOP_STEP / 2e-3 / 1e12)


def test_reference_arm_nonzero_rank_prints_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_warmup_below_three_rejected():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--warmup", "2"],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "warmup" in r.stderr
