"""Throughput of exact attention forward + backward on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c4] [--impl ours|reference]

A step is one pass of the whole path over one batch: fa_fwd, then fa_bwd (its three
kernels: delta preprocess, dK/dV pass, dQ pass). Inputs are seeded synthetic bf16 tensors
already resident in device memory when the timed region starts; they are larger than
the 126 MB L2 for the default workload, otherwise L2 is flushed before every timed step.
Under torchrun each rank runs its own replica of the workload on its own GPU (the
problems are independent: no collective on the data path); `value` is the flops of all
ranks divided by the slowest rank's time.

`--impl reference` times the fp64 CPU oracle instead (rank 0 only), each step a bounded
sample (a few (batch, head) pairs) of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd/fwd+bwd TFLOP/s, bf16 d=64/128, % of B200 dense BF16 peak"
DATASHEET_BF16_TFLOPS = 2250.0  # B200 dense bf16 (NVIDIA's sparse figure halved)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of a kernel on a
# workload, from one ncu capture of the kernels as they are now; an entry must be removed
# when its kernel changes. Compulsory traffic of the dK/dV pass on c4 is 537 MB read
# (Q, K, V, dO and the row statistics) and 268 MB written (dK, dV).
MEASURED_TRAFFIC = {
    ("c4_causal_b32h16n2048d64", "bwd_dkdv"): 792387840,
}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x10: "sync_boost"}

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._thread = None
        self._nvml = None
        self._index = device_index

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = self._index
            if vis:
                ids = [x for x in vis.split(",") if x.strip()]
                if idx < len(ids) and ids[idx].strip().isdigit():
                    idx = int(ids[idx])
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._sample()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception:  # NVML unavailable: clocks are reported as unknown
            self._nvml = None
        return self

    def _sample(self):
        nv = self._nvml
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        try:
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        except AttributeError:
            bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
        for b, name in self.REASONS.items():
            if bits & b:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.wait(self._period):
            try:
                self._sample()
            except Exception:
                break

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
            try:
                self._sample()
            except Exception:
                pass
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": sorted(self.reasons)}


# ------------------------------------------------------------------------- ranks
def max_over_ranks(value: float, dist, device) -> float:
    """The largest of `value` over all ranks (every rank gets it)."""
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the flops of every rank over the slowest rank's step time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------------- our arm
def run_ours(args, w, rank, world, local_rank):
    import torch

    from exact_attention_126_b200 import build, fa, synth, workloads

    build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    inp_host = synth.attention_inputs(w.B, w.H, w.N, w.d, w.seed_index, with_grad=True, pin=True)
    q, k, v, do = (inp_host[n].to(dev, non_blocking=True) for n in ("q", "k", "v", "do"))
    B, H, N, d = w.B, w.H, w.N, w.d
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
    scale = w.softmax_scale
    slopes = None
    if w.alibi:
        slopes = torch.tensor(workloads.alibi_slopes(H), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    inputs_bytes = 4 * w.tensor_bytes()
    flush = None
    if inputs_bytes <= L2_BYTES:
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def step(evs=None):
        # fa_fwd, then the three phases of fa_bwd, with optional events between kernels;
        # with ALiBi, fa_fwd_alibi and fa_bwd_alibi (the backward timed as one)
        if evs is not None:
            evs[0].record(stream)
        if w.alibi:
            fa.fa_fwd_alibi(q, k, v, o, lse, slopes, scale, w.causal, w.window, sp)
            if evs is not None:
                evs[1].record(stream)
            if w.backward:
                fa.fa_bwd_alibi(q, k, v, o, do, lse, dq, dk, dv, ws, slopes, scale, w.causal,
                                w.window, sp)
                if evs is not None:
                    evs[2].record(stream)
            return
        fa.fa_fwd(q, k, v, o, lse, scale, w.causal, w.window, sp)
        if evs is not None:
            evs[1].record(stream)
        if w.backward:
            fa.fa_bwd_preprocess(o, do, lse, ws, sp)
            if evs is not None:
                evs[2].record(stream)
            fa.fa_bwd_dkdv(q, k, v, do, ws, dk, dv, scale, w.causal, w.window, sp)
            if evs is not None:
                evs[3].record(stream)
            fa.fa_bwd_dq(q, k, v, do, ws, dq, scale, w.causal, w.window, sp)
            if evs is not None:
                evs[4].record(stream)

    n_ev = (3 if w.alibi else 5) if w.backward else 2
    launches_per_step = 4 if w.backward else 1

    for _ in range(args.warmup):
        if flush is not None:
            flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if fa.fa_debug_status(sp) != 0:
        raise RuntimeError("a kernel abandoned a bounded wait during warm-up")

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
              for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clocks:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for s in range(args.steps):
            if flush is not None:
                flush.zero_()
            step(events[s])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    if fa.fa_debug_status(sp) != 0:
        raise RuntimeError("a kernel abandoned a bounded wait in the timed region")

    # device time of the K steps (flushes excluded), and per kernel
    names = (["fwd", "bwd"] if w.alibi else ["fwd", "bwd_preprocess", "bwd_dkdv", "bwd_dq"])[
        : n_ev - 1]
    per_kernel = {n: 0.0 for n in names}
    step_ms = 0.0
    for evs in events:
        step_ms += evs[0].elapsed_time(evs[-1])
        for i, n in enumerate(names):
            per_kernel[n] += evs[i].elapsed_time(evs[i + 1])
    bracket_ms = t_start.elapsed_time(t_end)
    ms_per_step = step_ms / args.steps
    if flush is None:
        ms_per_step = bracket_ms / args.steps  # nothing but the steps in the bracket

    if dist is not None:
        ms_per_step = max_over_ranks(ms_per_step, dist, dev)

    # ---------------------------------------------------------------- end to end
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    host_out = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                for n, t in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv))}
    h2d_bytes = sum(inp_host[n].numel() * inp_host[n].element_size() for n in ("q", "k", "v", "do"))
    d2h_bytes = sum(t.numel() * t.element_size() for t in host_out.values())
    if not w.backward:
        h2d_bytes = sum(inp_host[n].numel() * inp_host[n].element_size() for n in ("q", "k", "v"))
        d2h_bytes = sum(host_out[n].numel() * host_out[n].element_size() for n in ("o", "lse"))

    def e2e_step():
        q.copy_(inp_host["q"], non_blocking=True)
        k.copy_(inp_host["k"], non_blocking=True)
        v.copy_(inp_host["v"], non_blocking=True)
        if w.backward:
            do.copy_(inp_host["do"], non_blocking=True)
        if w.alibi:
            fa.fa_fwd_alibi(q, k, v, o, lse, slopes, scale, w.causal, w.window, sp)
        else:
            fa.fa_fwd(q, k, v, o, lse, scale, w.causal, w.window, sp)
        host_out["o"].copy_(o, non_blocking=True)
        host_out["lse"].copy_(lse, non_blocking=True)
        if w.backward:
            dqq, dkk, dvv = fa.attention_backward(q, k, v, o, lse, do, scale, w.causal, w.window, sp,
                                                  alibi_slopes=slopes)
            host_out["dq"].copy_(dqq, non_blocking=True)
            host_out["dk"].copy_(dkk, non_blocking=True)
            host_out["dv"].copy_(dvv, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if dist is not None:
        e2e_ms = max_over_ranks(e2e_ms, dist, dev)
        dist.barrier()
        dist.destroy_process_group()

    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    flops = w.step_flops()
    value = job_tflops(flops, world, ms_per_step)
    kernel_flops = {"fwd": w.fwd_flops(), "bwd_preprocess": 0.0,
                    "bwd_dkdv": 2.0 * w.fwd_flops(), "bwd_dq": 0.5 * w.fwd_flops(),
                    "bwd": 2.5 * w.fwd_flops()}
    kernels = {}
    for n in names:
        avg = per_kernel[n] / args.steps
        kernels[n] = {"ms": round(avg, 5), "share": round(per_kernel[n] / step_ms, 4),
                      "algorithmic_tflops": round(kernel_flops[n] / (avg * 1e-3) / 1e12, 2)
                      if kernel_flops[n] else None}
    dominant = max(names, key=lambda n: per_kernel[n])
    dom_ms = per_kernel[dominant] / args.steps
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    if kernel_flops[dominant] > 0:
        achieved = kernel_flops[dominant] / (dom_ms * 1e-3) / 1e12
        roofline = {"kernel": dominant, "bound": "tensor", "achieved": round(achieved, 2),
                    "peak": sustained, "unit": "TFLOP/s", "frac": round(achieved / sustained, 4),
                    "peak_kind": "bf16 sustained (%s)" % peak_src,
                    "frac_of_burst": round(achieved / burst, 4),
                    "frac_of_datasheet": round(achieved / DATASHEET_BF16_TFLOPS, 4),
                    "traffic": MEASURED_TRAFFIC.get((w.name, dominant))}
    else:
        nbytes = w.bwd_bytes() if dominant.startswith("bwd") else w.fwd_bytes()
        achieved = 2 * w.tensor_bytes() / (dom_ms * 1e-3) / 1e9
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        roofline = {"kernel": dominant, "bound": "hbm", "achieved": round(achieved, 1),
                    "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                    "traffic": None, "compulsory_bytes": nbytes}
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded i.i.d. N(0,1) bf16, SplitMix64 + Box-Muller)",
        "config": {
            "workload": w.name, "B": B, "H": H, "N": N, "d": d, "causal": w.causal,
            "window": list(w.window), "alibi": w.alibi,
            "pass": "fwd+bwd" if w.backward else "fwd",
            "step_gflop": round(flops / 1e9, 3),
            "parallelism": "replicas" if world > 1 else "single",
            "l2": ("inputs larger than L2 (%d MB of inputs)" % (inputs_bytes >> 20))
            if flush is None else "L2 flushed before every timed step",
        },
        "pct_of_dense_peak": round(100 * value / world / DATASHEET_BF16_TFLOPS, 2),
        "pct_of_measured_peak": round(100 * value / world / burst, 2),
        "clocks": clocks.summary(),
        "e2e": {"value": round(job_tflops(flops, world, e2e_ms), 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 3), "steps": e2e_steps,
                "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes},
        "gpu_launches": launches_per_step * args.steps,
        "kernels": kernels,
        "roofline": roofline,
    }
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    return line


# ------------------------------------------------------------------------- CPU oracle
def _oracle_sample(w, b, h):
    """fp64 inputs of one (batch, head) problem of the workload (the same bf16 values the
    GPU arm uses)."""
    from exact_attention_126_b200 import synth
    x = synth.head_inputs(w.B, w.H, w.N, w.d, w.seed_index, b, h)
    return {n: synth.to_f64(t) for n, t in x.items()}


def _head_slope(w, h):
    """The ALiBi slope of head h as a one-head slope list for the oracle (None without)."""
    if not w.alibi:
        return None
    from exact_attention_126_b200 import workloads
    return [workloads.alibi_slopes(w.H)[h]]


def cpu_baseline(w, seconds: float):
    """Times the fp64 oracle, as it stands, on whole (batch, head) problems of the workload
    until `seconds` have passed (at least one head)."""
    import oracle
    orc = oracle.default()
    flops_per_head = w.step_flops() / (w.B * w.H)
    done, elapsed = 0, 0.0
    BH = w.B * w.H
    while elapsed < seconds and done < BH:
        b, h = divmod(done, w.H)
        x = _oracle_sample(w, b, h)
        slope = _head_slope(w, h)
        t0 = time.perf_counter()
        orc.fwd(x["q"], x["k"], x["v"], w.softmax_scale, w.causal, w.window, slope)
        if w.backward:
            orc.bwd(x["q"], x["k"], x["v"], x["do"], w.softmax_scale, w.causal, w.window, slope)
        elapsed += time.perf_counter() - t0
        done += 1
    return {"value": round(flops_per_head * done / elapsed / 1e12, 6), "unit": "TFLOP/s",
            "cores": orc.num_threads(), "kind": "oracle",
            "sample": "%d of %d (batch, head) problems of %s, fwd%s, %.1f s" % (
                done, BH, w.name, "+bwd" if w.backward else "", elapsed)}


def run_reference(args, w, rank):
    """The fp64 CPU oracle on the same workload: each step is one (batch, head) problem."""
    if rank != 0:
        return None
    import oracle
    orc = oracle.default()
    BH = w.B * w.H
    flops_per_head = w.step_flops() / BH
    heads_per_step = 1

    def one(idx):
        b, h = divmod(idx % BH, w.H)
        x = _oracle_sample(w, b, h)
        slope = _head_slope(w, h)
        t0 = time.perf_counter()
        orc.fwd(x["q"], x["k"], x["v"], w.softmax_scale, w.causal, w.window, slope)
        if w.backward:
            orc.bwd(x["q"], x["k"], x["v"], x["do"], w.softmax_scale, w.causal, w.window, slope)
        return time.perf_counter() - t0

    for i in range(args.warmup):
        one(i)
    total = sum(one(args.warmup + s) for s in range(args.steps))
    ms_per_step = total * 1e3 / args.steps
    value = flops_per_head * heads_per_step / (ms_per_step * 1e-3) / 1e12
    sample = "%d (batch, head) problem(s) of %s per step, fwd%s" % (
        heads_per_step, w.name, "+bwd" if w.backward else "")
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded i.i.d. N(0,1) bf16 widened to fp64)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "causal": w.causal, "window": list(w.window), "alibi": w.alibi,
                   "pass": "fwd+bwd" if w.backward else "fwd"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": orc.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="c4", help="c1, c2, c3, c4, c5c or c5w")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    from exact_attention_126_b200.workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, w, rank)
    else:
        line = run_ours(args, w, rank, world, local_rank)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
