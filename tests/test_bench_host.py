"""bench.py's host logic without a GPU: the max-over-ranks timing on two gloo ranks, the
whole-job throughput formula, and the reference arm's JSON line (the fp64 oracle on CPU)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    # rank r measured (r + 1) * 10 ms per step: the job is as slow as its slowest rank
    ms = bench.max_over_ranks(10.0 * (rank + 1), dist, torch.device("cpu"))
    out[rank] = ms
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_on_two_gloo_ranks():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert dict(out) == {0: 20.0, 1: 20.0}


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # two replicas of 1 TFLOP each, slowest rank 100 ms per step -> 20 TFLOP/s for the job
    assert bench.job_tflops(1e12, 2, 100.0) == pytest.approx(20.0)


def test_reference_arm_json_line():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--workload", "c1", "--steps", "2", "--warmup", "3"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert res.returncode == 0, res.stderr
    line = json.loads(res.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0


def test_reference_arm_other_ranks_do_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--workload", "c1", "--steps", "1", "--warmup", "3"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert res.returncode == 0 and res.stdout.strip() == ""


def test_roofline_peak_follows_the_timed_region():
    """Regions under a second are held to the burst peak, longer ones to the sustained."""
    sys.path.insert(0, ROOT)
    import bench
    peaks = {"bf16_tflops": 1679.8, "bf16_tflops_sustained": 1394.0}
    assert bench.roofline_peak(peaks, 47.0)[:2] == (1679.8, "burst")
    assert bench.roofline_peak(peaks, 2500.0)[:2] == (1394.0, "sustained")
    assert bench.roofline_peak({}, 10.0)[0] == bench.FALLBACK_PEAKS["bf16_tflops"]


def test_traffic_is_null_once_the_kernels_change(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    h = bench.kernel_source_hash("k")
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", {
        ("w", "k"): (123, h, "ncu capture"), ("w", "old"): (456, "0" * 12, "old capture")})
    assert bench.measured_traffic("w", "k") == (123, "ncu capture")
    assert bench.measured_traffic("w", "old") == (None, None)
    assert bench.measured_traffic("w", "none") == (None, None)


def test_traffic_hash_covers_only_the_kernels_sources():
    """A kernel's traffic figure depends on the shared headers and its own sources only."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.kernel_source_hash("bwd_dkdv") == bench.kernel_source_hash("bwd_dq")
    assert bench.kernel_source_hash("bwd_dkdv") != bench.kernel_source_hash("fwd")
    assert bench.kernel_source_hash() not in (bench.kernel_source_hash("fwd"),
                                              bench.kernel_source_hash("bwd_dkdv"))
