"""The multi-GPU bench path, exercised with world_size-2 gloo ranks on CPU.

Each GPU runs its own copy of the workload (the heads of attention are
independent, so nothing crosses between GPUs on the data path).  What the
ranks share is bookkeeping: every rank draws its own seeded inputs of the same
shape, the timing is the slowest rank's, and the reported throughput is all
ranks' FLOPs over that time.
"""

from __future__ import annotations

import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    from exact_io_aware_51_b200 import inputs as I
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # per-rank inputs: same shape, different seed
        qi, ki, vi, doi = I.make_inputs(1, 64, 2, 64, seed=rank)
        shapes = dist_gather_obj((tuple(qi.shape), float(qi.float().sum())), world)
        # the slowest rank's time is everybody's time
        local_ms = 10.0 + 5.0 * rank
        slow = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        value = bench.aggregate_tflops(3.5e12, steps=4, world=world, ms_max=slow)
        q.put((rank, shapes, slow, value))
    finally:
        dist.destroy_process_group()


def dist_gather_obj(obj, world):
    out = [None] * world
    dist.all_gather_object(out, obj)
    return out


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, shapes, slow, value in res:
        assert slow == 15.0
        # 2 ranks x 4 steps x 3.5 TFLOP over 15 ms
        assert value == pytest.approx(2 * 4 * 3.5 / 15e-3)
        assert shapes[0][0] == shapes[1][0]          # same shape on every rank
        assert shapes[0][1] != shapes[1][1]          # but each rank's own inputs


def test_reference_arm_on_a_non_zero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_clock_scaled_fraction():
    """The fraction at the maximum SM clock is frac x max MHz / median MHz, and
    None when there is no clock record."""
    sys.path.insert(0, ROOT)
    import bench
    assert abs(bench.clock_scaled(0.6, {"sm_mhz": 1700.0, "sm_max_mhz": 1965.0}) - 0.6 * 1965 / 1700) < 1e-12
    assert bench.clock_scaled(0.6, {"sm_mhz": None, "sm_max_mhz": 1965.0}) is None
    assert bench.clock_scaled(0.6, {}) is None
    assert bench.clock_scaled(0.6, None) is None


def test_nvml_sampler_keeps_only_the_marked_window():
    """Samples outside [mark_begin, mark_end] are dropped; no samples gives None."""
    sys.path.insert(0, ROOT)
    import bench
    s = bench.NvmlSampler(0)

    class _T:  # stands in for the sampling thread that ran
        def join(self, timeout=None):
            return None
    s.thread = _T()
    s.max_mhz = 1965
    s.begin, s.end = 10.0, 20.0
    s.rows = [(5.0, 1965, 300.0, 0), (12.0, 1700, 900.0, 0x4), (15.0, 1690, 950.0, 0x4), (25.0, 1965, 200.0, 0)]
    r = s.stop()
    assert r["samples"] == 2 and r["sm_mhz"] == 1695 and r["reasons"] == ["sw_power_cap"]
    s2 = bench.NvmlSampler(0)
    assert s2.stop() is None


def test_reference_arm_prints_the_contract_line():
    """Rank 0 of the reference arm (the CPU oracle) prints one JSON line with the
    keys the bench contract asks for, its own e2e object and a cpu_baseline."""
    import json
    env = dict(os.environ, RANK="0", LOCAL_RANK="0", WORLD_SIZE="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["impl"] == "reference" and j["value"] > 0 and j["cpu_baseline"]["kind"] == "oracle"
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["value"] == j["value"]
