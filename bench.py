#!/usr/bin/env python
"""Attention TFLOP/s on B200: fused forward + recomputing backward, bf16.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole hot path over one batch of synthetic input:
the fused forward (O and LSE) followed by the backward (preprocess, main
kernel, dQ conversion) producing dQ, dK and dV.  Workload: bf16 B=1, H=32,
N=16384, d=128, non-causal, Q/K/V/dO i.i.d. N(0,1) with 1% of K rows scaled by
3 (seeded; one seed per rank).  Every tensor is 128 MiB, larger than the L2,
so no flush is needed between steps.

Throughput counts 4*B*H*N^2*d FLOPs for the forward and 2.5x that for the
backward; `value` = all ranks' FLOPs / the slowest rank's device time for K
steps (CUDA events on the launching stream, barrier + synchronize on both
sides).  With --gpus N > 1 (launched by torchrun) each rank runs its own copy
of the workload: the problem shards into independent (b, h) heads, so there is
no collective on the data path (weak scaling).

--impl reference times the CPU oracle (fp64, materialises S and P) on the
host cores: each step is one (b, h) head of the same workload, forward and
backward; rank 0 alone runs it.

Prints one JSON line.
"""

from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import pathlib
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = pathlib.Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "attention TFLOP/s (fwd, fwd+bwd) bf16 on 1 B200 and % of dense BF16 tensor peak"
WORKLOAD = dict(B=1, H=32, N=16384, d=128, causal=False, spike_frac=0.01, spike=3.0)
DECODE_WORKLOAD = dict(B=64, H=64, Hkv=8, d=128, page=16, lo=512, hi=8192, seed=21)
DECODE_NAME = "bf16 paged decode B64 H64 Hkv8 d128, 16-token pages, lengths 512..8192"
WORKLOAD_NAME = "bf16 fwd+bwd B1 H32 N16384 d128 non-causal, K rows x3 at 1% of positions"
FALLBACK_PEAK_TFLOPS = 1590.0  # earlier burst measurement of cuBLAS bf16 on this machine


def flops_fwd(B, H, N, d, causal):
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def read_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        j = json.loads(p.read_text())
        return float(j["bf16_tflops"]), float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), "measured"
    return FALLBACK_PEAK_TFLOPS, 1400.0, "fallback"


SPEC_PEAK_TFLOPS = 2250.0  # B200 dense BF16 tensor-core figure (public spec), for context beside the measured one


def clock_scaled(frac: float, clocks: dict) -> float | None:
    """The fraction the same kernel would reach at the maximum SM clock: frac x
    max MHz / median MHz over the timed window (None without a clock record)."""
    mhz, top = (clocks or {}).get("sm_mhz"), (clocks or {}).get("sm_max_mhz")
    return frac * float(top) / float(mhz) if mhz and top else None


def read_hbm_peak():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        return float(json.loads(p.read_text())["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def read_profile_traffic(kernel_key: str):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current source."""
    prof = ROOT / "profiles" / {"fwd_bf16": "fwd_bf16_b1_h32_n16384_d128.md",
                                "bwd_main": "bwd_main_b1_h32_n16384_d128.md"}[kernel_key]
    if not prof.exists():
        return None
    text = prof.read_text()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"source_sha256:\s*([0-9a-f]+)", text)
    if not m or not h:
        return None
    import hashlib
    src = {"fwd_bf16": "fa_fwd_bf16.cu", "bwd_main": "fa_bwd.cu"}[kernel_key]
    cur = hashlib.sha256((ROOT / "exact_io_aware_51_b200" / "csrc" / src).read_bytes()).hexdigest()
    return float(m.group(1)) if cur.startswith(h.group(1)) else None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the GPU is busy."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.5)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in pathlib.Path(self.path).read_text().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r[2] > 250.0] or rows
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(loaded)}


class NvmlSampler:
    """In-process NVML sampling (every 5 ms) of the SM clock, power and clock-event
    reasons, kept only for the window between mark_begin() and mark_end(), which
    bracket the timed region on the host (the stream is synchronised at both ends)."""

    REASONS = ((0x4, "sw_power_cap"), (0x8, "hw_slowdown"), (0x20, "sw_thermal_slowdown"),
               (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown"))

    def __init__(self, index: int):
        self.index, self.rows, self.thread, self.begin, self.end = index, [], None, None, None
        self.stop_flag = False

    def start(self):
        try:
            import threading

            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - no NVML: the nvidia-smi record stands alone
            return

        def body():
            while not self.stop_flag:
                try:
                    self.rows.append((time.perf_counter(), pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                      pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                      pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)))
                except Exception:  # noqa: BLE001
                    return
                time.sleep(0.005)

        self.thread = threading.Thread(target=body, daemon=True)
        self.thread.start()

    def mark_begin(self):
        self.begin = time.perf_counter()

    def mark_end(self):
        self.end = time.perf_counter()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join(timeout=5)
        return self.window(self.begin, self.end)

    def window(self, begin, end):
        """Clock statistics over the samples taken between two perf_counter() marks."""
        rows = [r for r in self.rows if begin is not None and end is not None and begin <= r[0] <= end]
        if not rows:
            return None
        bits = 0
        for r in rows:
            bits |= r[3]
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_min_mhz": min(r[1] for r in rows),
                "sm_max_mhz": float(self.max_mhz), "power_w_median": statistics.median(r[2] for r in rows),
                "reasons": [name for bit, name in self.REASONS if bits & bit], "samples": len(rows),
                "how": "NVML every 5 ms, in-process, over exactly the timed region"}


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n and n[0]:
            return int(n[0])
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_head_step(q, k, v, do, scale, causal):
    """Time the CPU oracle on one (b, h) head: forward then backward."""
    import oracle
    t0 = time.perf_counter()
    oracle.forward_head(q, k, v, scale, causal)
    oracle.backward_head(q, k, v, do, scale, causal)
    return time.perf_counter() - t0


def head_inputs(seed=0):
    import numpy as np
    from exact_io_aware_51_b200 import inputs as I
    w = WORKLOAD
    q, k, v, do = I.make_inputs(w["B"], w["N"], w["H"], w["d"], seed=seed, spike_frac=w["spike_frac"],
                                spike=w["spike"])
    return tuple(t[0, :, 0].float().numpy().astype(np.float64) for t in (q, k, v, do))


def max_over_ranks(x: float, dist=None, device=None) -> float:
    """The slowest rank's value (all ranks take part; a no-op without a process group)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flops_per_rank_step: float, steps: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's FLOPs over the slowest rank's time."""
    return flops_per_rank_step * steps * world / (ms_max * 1e-3) / 1e12


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def run_reference(args, world, rank):
    if rank != 0:
        return None
    w = WORKLOAD
    scale = float(1.0 / math.sqrt(w["d"]))
    q, k, v, do = head_inputs(0)
    for _ in range(args.warmup):
        oracle_head_step(q, k, v, do, scale, w["causal"])
    times = [oracle_head_step(q, k, v, do, scale, w["causal"]) for _ in range(args.steps)]
    f_head = flops_fwd(1, 1, w["N"], w["d"], w["causal"])
    tot = sum(times)
    value = 3.5 * f_head * args.steps / tot / 1e12
    cores = cpu_cores()
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_NAME, **w, "sample": "one (b, h) head per step"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": "forward + backward of one (b, h) head (N=16384, d=128) per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_sweep(fa, I, dev, stream, main, peak, nvml):
    """Every problem family of the method, timed with CUDA events after the
    headline region: each entry is a short loop of launches (3 warm-ups, then
    enough launches for about 30 ms, at least 10) of the forward, or of the
    forward followed by the backward, on seeded inputs of that family's shapes.
    The clock record of each loop gives the fraction scaled to the maximum SM
    clock.  Parity of every entry is the GPU test suite's job; nothing here
    checks values."""
    import torch

    def timed(fwd, bwd, n_min=10, target_ms=30.0):
        evs = lambda: torch.cuda.Event(enable_timing=True)
        for _ in range(3):
            fwd()
            if bwd:
                bwd()
        e0, e1 = evs(), evs()
        e0.record(stream)
        fwd()
        if bwd:
            bwd()
        e1.record(stream)
        torch.cuda.synchronize()
        n = max(n_min, min(200, math.ceil(target_ms / max(e0.elapsed_time(e1), 1e-3))))
        marks = [(evs(), evs(), evs()) for _ in range(n)]
        t_begin = time.perf_counter()
        for a, b, c in marks:
            a.record(stream)
            fwd()
            b.record(stream)
            if bwd:
                bwd()
            c.record(stream)
        torch.cuda.synchronize()
        t_end = time.perf_counter()
        f_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in marks)
        b_ms = statistics.mean(b.elapsed_time(c) for _, b, c in marks) if bwd else None
        clk = nvml.window(t_begin, t_end) if nvml is not None else None
        return f_ms, b_ms, n, clk

    def entry(w, causal, with_bwd, tensors=None):
        if tensors is None:
            q, k, v, do = I.make_inputs(w.B, w.N, w.H, w.d, seed=w.seed, dtype=w.dtype, spike_frac=w.spike_frac,
                                        spike=w.spike, with_do=with_bwd, kv_heads=w.Hkv or None)
            q, k, v = (t.to(dev) for t in (q, k, v))
            do = do.to(dev) if with_bwd else None
        else:
            q, k, v, do = tensors
        sc = float(1.0 / math.sqrt(w.d))
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
        bufs = {}
        if with_bwd:
            bufs = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                        workspace=torch.empty(fa.bwd_workspace_size(w.B, w.H, w.N, w.d, kv_heads=w.kv_heads),
                                              dtype=torch.uint8, device=dev))
        fwd = lambda: fa.fwd(q, k, v, causal=causal, scale=sc, out=o, lse=lse)
        bwd = (lambda: fa.bwd(q, k, v, o, do, lse, causal=causal, scale=sc, **bufs)) if with_bwd else None
        f_ms, b_ms, n, clk = timed(fwd, bwd)
        F = w.flops_fwd(causal)
        r = {"workload": w.name, "causal": causal, "launches": n, "fwd_ms": f_ms, "fwd_tflops": F / f_ms / 1e9}
        if w.dtype == "bf16":
            r["fwd_frac"] = r["fwd_tflops"] / peak
        if with_bwd:
            r.update(bwd_ms=b_ms, bwd_tflops=2.5 * F / b_ms / 1e9, fwdbwd_tflops=3.5 * F / (f_ms + b_ms) / 1e9)
            r["bwd_frac"] = r["bwd_tflops"] / peak
            r["fwdbwd_frac"] = r["fwdbwd_tflops"] / peak
        if clk is not None:
            r["sm_mhz"] = clk["sm_mhz"]
            r["reasons"] = clk["reasons"]
            if "fwd_frac" in r:
                r["fwd_frac_at_max_clock"] = clock_scaled(r["fwd_frac"], clk)
            if with_bwd:
                r["fwdbwd_frac_at_max_clock"] = clock_scaled(r["fwdbwd_frac"], clk)
        return r

    out = [entry(I.FP32_SMALL, False, False)]
    out += [entry(I.BF16_FWD_N1K, c, False) for c in (False, True)]
    out.append(entry(I.BF16_FWDBWD_N4K, True, True))
    out.append(entry(I.BF16_FWDBWD_N16K, True, True, tensors=main))
    out.append(entry(I.BF16_FWDBWD_N16K, False, False, tensors=main))
    out.append(entry(I.BF16_FWDBWD_N16K_D64, False, True))  # the d = 64 backward kernel
    for w in I.SWEEP:
        out += [entry(w, c, False) for c in (False, True)]
    out += [entry(I.BF16_GQA_H64_KV8, c, True) for c in (False, True)]
    return {"how": "CUDA events around each launch, short loops after the headline region; fractions of the "
                   "measured burst cuBLAS figure; *_at_max_clock scales by max / median SM MHz over the loop",
            "peak": peak, "entries": out}


def run_ours(args, world, rank, local):
    import torch

    import exact_io_aware_51_b200 as fa
    from exact_io_aware_51_b200 import inputs as I

    dist = None
    if world > 1:
        import torch.distributed as dist
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = WORKLOAD
    B, H, N, d, causal = w["B"], w["H"], w["N"], w["d"], w["causal"]
    scale = float(1.0 / math.sqrt(d))
    q_h, k_h, v_h, do_h = I.make_inputs(B, N, H, d, seed=rank, spike_frac=w["spike_frac"], spike=w["spike"])
    q, k, v, do = (t.to(dev) for t in (q_h, k_h, v_h, do_h))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.fwd(q, k, v, causal=causal, scale=scale, out=o, lse=lse)
        fa.bwd(q, k, v, o, do, lse, causal=causal, scale=scale, workspace=ws, dq=dq, dk=dk, dv=dv)

    def barrier():
        if dist is not None:
            dist.barrier()

    def slowest(x: float) -> float:
        return max_over_ranks(x, dist, dev)

    # ---- timed region: K steps, kernel events around the two tensor-core kernels ----
    def kernel_event():
        # torch creates the CUDA event lazily on its first record; record it once
        # here so the handle exists when the library records it around a kernel
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        return e

    ev_f = [(kernel_event(), kernel_event()) for _ in range(args.steps)]
    ev_b = [(kernel_event(), kernel_event()) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # the samplers start first, so the warm-up steps lead straight into the timed
    # ones with no idle gap: the timed steps run in the same power state as a
    # continuous training loop (on this part, at the power cap)
    sampler, fine = ClockSampler(local), NvmlSampler(local)
    sampler.start()
    fine.start()
    for _ in range(args.warmup):
        step()
    barrier()
    torch.cuda.synchronize()
    fine.mark_begin()
    t0.record(stream)
    for i in range(args.steps):
        fa.set_kernel_events(*ev_f[i])
        fa.fwd(q, k, v, causal=causal, scale=scale, out=o, lse=lse)
        fa.set_kernel_events(*ev_b[i])
        fa.bwd(q, k, v, o, do, lse, causal=causal, scale=scale, workspace=ws, dq=dq, dk=dk, dv=dv)
    fa.set_kernel_events(None, None)
    t1.record(stream)
    torch.cuda.synchronize()
    fine.mark_end()
    barrier()
    clocks = sampler.stop()
    fine_clocks = fine.stop()
    if fine_clocks is not None:
        # the 5 ms NVML record covers exactly the timed region; the nvidia-smi one
        # (100 ms) is kept beside it
        clocks = {**fine_clocks, "nvidia_smi": clocks}
    rc, detail = fa.last_device_status()
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail:#x}) after the timed region")
    ms_local = t0.elapsed_time(t1)
    ms = slowest(ms_local)
    fwd_ms = slowest(statistics.mean(a.elapsed_time(b) for a, b in ev_f))
    bwd_main_ms = slowest(statistics.mean(a.elapsed_time(b) for a, b in ev_b))

    f = flops_fwd(B, H, N, d, causal)
    value = aggregate_tflops(3.5 * f, args.steps, world, ms)
    ms_step = ms / args.steps
    peak_burst, peak_sustained, peak_src = read_peaks()
    fwd_tflops = f / (fwd_ms * 1e-3) / 1e12
    bwd_main_tflops = 2.5 * f / (bwd_main_ms * 1e-3) / 1e12
    bwd_total_ms = ms_step - fwd_ms  # preprocess + main + dQ convert

    # dominant kernel of the step
    if bwd_main_ms >= fwd_ms:
        dom = {"kernel": "bwd_main_kernel", "flops": 2.5 * f, "ms": bwd_main_ms, "key": "bwd_main"}
    else:
        dom = {"kernel": "fwd_bf16_kernel", "flops": f, "ms": fwd_ms, "key": "fwd_bf16"}
    achieved = dom["flops"] / (dom["ms"] * 1e-3) / 1e12
    # The fraction is taken against the measured burst cuBLAS figure.  The steps
    # run at the power cap, so the fraction scaled to the maximum SM clock is
    # given beside it, and the sustained-peak and spec-peak fractions for context.
    peak = peak_burst
    frac = achieved / peak
    roofline = {"bound": "tensor", "kernel": dom["kernel"], "achieved": achieved, "peak": peak,
                "peak_source": f"{peak_src} bf16 burst (cuBLAS)", "unit": "TFLOP/s", "frac": frac,
                "frac_at_max_clock": clock_scaled(frac, clocks),
                "frac_of_sustained": achieved / peak_sustained, "frac_of_spec": achieved / SPEC_PEAK_TFLOPS,
                "traffic": read_profile_traffic(dom["key"]),
                "flops_per_launch": dom["flops"], "ms_per_launch": dom["ms"]}

    # ---- the 8-bit forward on the same workload (e4m3 codes, per-tensor scales) ----
    fp8 = None
    if hasattr(torch, "float8_e4m3fn"):
        codes, scales = [], []
        for t in (q, k, v):
            s_t = float(t.float().abs().max()) / 448.0 or 1.0
            codes.append((t.float() / s_t).to(torch.float8_e4m3fn))
            scales.append(s_t)
        o8 = torch.empty_like(o)
        for _ in range(3):
            fa.fwd_fp8(*codes, *scales, causal=causal, scale=scale, out=o8, lse=lse)
        n8 = max(3, min(args.steps, 10))
        e8a, e8b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clk8 = NvmlSampler(local)  # the leg follows the power-capped region: record its own clock
        clk8.start()
        barrier()
        torch.cuda.synchronize()
        clk8.mark_begin()
        e8a.record(stream)
        for _ in range(n8):
            fa.fwd_fp8(*codes, *scales, causal=causal, scale=scale, out=o8, lse=lse)
        e8b.record(stream)
        torch.cuda.synchronize()
        clk8.mark_end()
        barrier()
        c8 = clk8.stop()
        ms8 = slowest(e8a.elapsed_time(e8b)) / n8
        tf8 = f / (ms8 * 1e-3) / 1e12
        fp8 = {"tflops": tf8, "ms": ms8, "launches": n8, "peak": 2 * peak_burst,
               "frac_of_peak": tf8 / (2 * peak_burst),
               "frac_at_max_clock": clock_scaled(tf8 / (2 * peak_burst), c8),
               "sm_mhz": (c8 or {}).get("sm_mhz"), "reasons": (c8 or {}).get("reasons"),
               "peak_source": "bf16 burst x 2 (the nominal e4m3 / bf16 dense ratio)",
               "inputs": "Q, K, V of the same workload as e4m3 codes with per-tensor scales"}
        del codes, o8

    # ---- one decode step over a paged KV cache (HBM-bound; its own workload) ----
    # 64 sequences, 64 query heads on 8 K/V heads, d 128, 16-token pages handed
    # out in shuffled order, lengths uniform in [512, 8192]: 1.16 GB of K/V per
    # step, larger than L2.
    dw = DECODE_WORKLOAD
    dlens = I.decode_lengths(dw["B"], dw["lo"], dw["hi"], seed=dw["seed"] + rank)
    dq_, dk_, dv_, dt_, ds_ = (t.to(dev) for t in I.make_paged_decode(
        dw["B"], dw["H"], dw["Hkv"], dw["d"], dw["page"], dlens, seed=dw["seed"] + rank))
    dws = torch.empty(max(1, fa.decode_workspace_size(dw["B"], dw["H"], dw["Hkv"], dw["d"], dw["page"],
                                                      dt_.shape[1])), dtype=torch.uint8, device=dev)
    d_o, d_l = fa.decode_paged(dq_, dk_, dv_, dt_, ds_, workspace=dws)
    for _ in range(5):
        fa.decode_paged(dq_, dk_, dv_, dt_, ds_, out=d_o, lse=d_l, workspace=dws)
    nd = max(5, min(4 * args.steps, 50))
    ed0, ed1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    ed0.record(stream)
    for _ in range(nd):
        fa.decode_paged(dq_, dk_, dv_, dt_, ds_, out=d_o, lse=d_l, workspace=dws)
    ed1.record(stream)
    torch.cuda.synchronize()
    barrier()
    rc, detail = fa.last_device_status()
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail:#x}) after the decode steps")
    d_ms = slowest(ed0.elapsed_time(ed1)) / nd
    d_bytes = (sum(dlens) * dw["Hkv"] * dw["d"] * 2 * 2 + 2 * dw["B"] * dw["H"] * dw["d"] * 2
               + dw["B"] * dw["H"] * 4 + dw["B"] * (dt_.shape[1] + 1) * 4)
    hbm, hbm_src = read_hbm_peak()
    decode = {"workload": DECODE_NAME, "gbs": d_bytes / (d_ms * 1e-3) / 1e9, "us": d_ms * 1e3, "launches": nd,
              "bytes_per_launch": d_bytes, "bound": "hbm", "peak_gbs": hbm, "peak_source": f"{hbm_src} copy",
              "frac_of_peak": d_bytes / (d_ms * 1e-3) / 1e9 / hbm,
              "bytes": "K and V rows of every cached position once, Q and O, LSE, block table and lengths"}
    del dq_, dk_, dv_, dt_, ds_, dws, d_o, d_l

    # ---- end to end through the public API with host buffers ----
    # Every step copies its four inputs from pinned host memory and its five
    # outputs back.  Two device buffer sets and two copy streams pipeline the
    # steps: the inputs of step s+1 go up and the outputs of step s-1 come down
    # while step s computes.
    pin = [t.pin_memory() for t in (q_h, k_h, v_h, do_h)]
    out_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (o, lse, dq, dk, dv)]
    h2d = sum(t.numel() * t.element_size() for t in pin)
    d2h = sum(t.numel() * t.element_size() for t in out_h)
    e_steps = max(1, args.steps)  # as many steps as the device-timed region: fill and drain amortise alike
    bufs = [dict(q=q, k=k, v=v, do=do, o=o, lse=lse, dq=dq, dk=dk, dv=dv)]
    bufs.append({key: torch.empty_like(t) for key, t in bufs[0].items()})
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()

    def e2e_run(n_steps):
        inputs_in = [ev(), ev()]      # H2D of a buffer set finished
        computed = [ev(), ev()]       # compute on a buffer set finished
        drained = [ev(), ev()]        # D2H of a buffer set finished
        started = ev()
        started.record(stream)

        def upload(i):
            bset = bufs[i % 2]
            up.wait_event(started)
            if i >= 2:
                up.wait_event(computed[i % 2])  # step i-2 has finished reading this set
            with torch.cuda.stream(up):
                for key, src in zip(("q", "k", "v", "do"), pin):
                    bset[key].copy_(src, non_blocking=True)
            inputs_in[i % 2].record(up)

        upload(0)
        for i in range(n_steps):
            bset = bufs[i % 2]
            if i + 1 < n_steps:
                upload(i + 1)
            stream.wait_event(inputs_in[i % 2])
            if i >= 2:
                stream.wait_event(drained[i % 2])  # outputs of step i-2 are on the host
            fa.fwd(bset["q"], bset["k"], bset["v"], causal=causal, scale=scale, out=bset["o"], lse=bset["lse"])
            fa.bwd(bset["q"], bset["k"], bset["v"], bset["o"], bset["do"], bset["lse"], causal=causal, scale=scale,
                   workspace=ws, dq=bset["dq"], dk=bset["dk"], dv=bset["dv"])
            computed[i % 2].record(stream)
            down.wait_event(computed[i % 2])
            with torch.cuda.stream(down):
                for dst, key in zip(out_h, ("o", "lse", "dq", "dk", "dv")):
                    dst.copy_(bset[key], non_blocking=True)
            drained[i % 2].record(down)
        stream.wait_event(drained[(n_steps - 1) % 2])
        if n_steps >= 2:
            stream.wait_event(drained[(n_steps - 2) % 2])

    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = slowest(e0.elapsed_time(e1))
    e2e_value = aggregate_tflops(3.5 * f, e_steps, world, e2e_ms)

    sweep = None
    if not args.no_sweep:
        sweep_clocks = NvmlSampler(local)
        sweep_clocks.start()
        sweep = run_sweep(fa, I, dev, stream, (q, k, v, do), peak,
                          sweep_clocks if sweep_clocks.thread is not None else None)
        sweep_clocks.stop()
        rc, detail = fa.last_device_status()
        if rc != 0:
            raise RuntimeError(f"device status {rc} ({detail:#x}) after the sweep")

    result = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_NAME, "B": B, "H": H, "N": N, "d": d, "causal": causal,
                   "global_batch": B * world, "seq_len": N,
                   "parallelism": f"replicas: one independent workload per GPU ({world})",
                   "l2": "inputs larger than L2 (each of Q, K, V, O, dO is 128 MiB); no flush"},
        "fwd": {"tflops": fwd_tflops, "frac_of_peak": fwd_tflops / peak,
                "frac_at_max_clock": clock_scaled(fwd_tflops / peak, clocks),
                "frac_of_spec": fwd_tflops / SPEC_PEAK_TFLOPS, "ms": fwd_ms},
        "bwd": {"tflops": 2.5 * f / (bwd_total_ms * 1e-3) / 1e12, "ms": bwd_total_ms,
                "main_kernel_tflops": bwd_main_tflops, "main_kernel_ms": bwd_main_ms,
                "main_frac_of_peak": bwd_main_tflops / peak,
                "main_frac_at_max_clock": clock_scaled(bwd_main_tflops / peak, clocks),
                "main_frac_of_spec": bwd_main_tflops / SPEC_PEAK_TFLOPS},
        "frac_of_peak": value / world / peak,
        "frac_of_spec": value / world / SPEC_PEAK_TFLOPS,
        "peak_tflops": {"burst": peak_burst, "sustained": peak_sustained, "used": peak, "source": peak_src,
                        "spec": SPEC_PEAK_TFLOPS,
                        "note": "fractions are of the measured burst cuBLAS figure unless named otherwise"},
        "roofline": roofline,
        "fwd_fp8": fp8,
        "decode_paged": decode,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e_steps, "ms_per_step": e2e_ms / e_steps,
                "how": "pinned host -> device inputs and device -> pinned host outputs every step, "
                       "pipelined over two device buffer sets on separate copy streams"},
        "sweep": sweep,
        "gpu_launches": 4 * args.steps,
        "clocks": clocks,
    }
    del pin, out_h, bufs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        qh, kh, vh, doh = (t[0, :, 0].float().numpy().astype("float64") for t in (q_h, k_h, v_h, do_h))
        t = oracle_head_step(qh, kh, vh, doh, scale, causal)
        result["cpu_baseline"] = {
            "value": 3.5 * flops_fwd(1, 1, N, d, causal) / t / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(),
            "kind": "oracle", "sample": "forward + backward of one (b, h) head (N=16384, d=128), fp64",
            "seconds": t}
    return result


PROFILE_WORKLOAD = dict(B=1, H=64, N=4096, d=128)


def run_profile_case(args):
    """Small case for ncu section captures: 2 x (forward, backward) on B1 H64 N4096 d128
    (each tensor 64 MiB, so the five of them exceed the L2; < 1 GB on the device), then
    2 x the 8-bit forward on the same Q, K, V.  With --profile-d64: the same at d = 64
    (32 MiB tensors, five of them still beyond the L2), without the 8-bit forward."""
    import torch

    import exact_io_aware_51_b200 as fa
    from exact_io_aware_51_b200 import inputs as I
    w = dict(PROFILE_WORKLOAD, d=64) if args.profile_d64 else PROFILE_WORKLOAD
    q, k, v, do = (t.cuda() for t in I.make_inputs(w["B"], w["N"], w["H"], w["d"], seed=0))
    for causal in ((False, True) if args.profile_causal else (False,)):
        for _ in range(2):
            o, lse = fa.fwd(q, k, v, causal=causal)
            fa.bwd(q, k, v, o, do, lse, causal=causal)
    if w["d"] == 128:
        q8, k8, v8 = (t.to(torch.float8_e4m3fn) for t in (q, k, v))
        for _ in range(2):
            fa.fwd_fp8(q8, k8, v8, 1.0, 1.0, 1.0)
    torch.cuda.synchronize()
    rc, detail = fa.last_device_status()
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail:#x})")
    print(json.dumps({"profile_case": w, "ok": True}))


def run_profile_decode():
    """Small case for ncu section captures of the paged decode: 2 launches on 32
    sequences (lengths 512..8192, 64 query heads on 8 K/V heads, d 128, 16-token
    pages): about 0.6 GB of K/V, more than the L2, well under the device memory."""
    import torch

    import exact_io_aware_51_b200 as fa
    from exact_io_aware_51_b200 import inputs as I
    lens = I.decode_lengths(32, 512, 8192, seed=21)
    q, k, v, t, s = (x.cuda() for x in I.make_paged_decode(32, 64, 8, 128, 16, lens, seed=21))
    for _ in range(2):
        fa.decode_paged(q, k, v, t, s)
    torch.cuda.synchronize()
    rc, detail = fa.last_device_status()
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail:#x})")
    print(json.dumps({"profile_case": "decode B32 H64 Hkv8 d128 P16", "ok": True}))


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing on the host")
    ap.add_argument("--no-sweep", action="store_true", help="skip the per-family timing loops after the headline")
    ap.add_argument("--profile-case", action="store_true",
                    help="run only the small profiling case (2 x fwd + bwd, B1 H64 N4096 d128) for ncu")
    ap.add_argument("--profile-causal", action="store_true", help="with --profile-case: also the causal pair")
    ap.add_argument("--profile-d64", action="store_true",
                    help="with --profile-case: d = 64 instead of 128 (B1 H64 N4096 d64, no 8-bit forward)")
    ap.add_argument("--profile-decode", action="store_true",
                    help="run only the small paged-decode profiling case (2 launches, B32) for ncu")
    args = ap.parse_args()
    if args.profile_decode:
        run_profile_decode()
        return
    if args.profile_case:
        run_profile_case(args)
        return
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            res = run_reference(args, world, rank)
        else:
            res = run_ours(args, world, rank, local)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1 and args.impl == "ours":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
