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
# workload, from one ncu capture, with the SHA-256 of the sources that kernel was built from
# (kernel_source_hash(kernel)); an entry whose hash no longer matches is reported as null.
MEASURED_TRAFFIC = {
    ("c4_causal_b32h16n2048d64", "fwd"): (639792640, "0bb51163869f",
                                          "ncu --set full, one launch"),
    ("c5_causal_b2h32n8192d128", "fwd"): (647730944, "0bb51163869f",
                                          "ncu --set full, one launch"),
    ("c4_causal_varlen_b32h16n2048d64", "fwd"): (778232576, "0bb51163869f",
                                                 "ncu --set full, one launch"),
    ("c4_causal_packed_b32h16n2048d64", "fwd"): (748935168, "0bb51163869f",
                                                 "ncu --set full, one launch"),
    ("c4_causal_b32h16n2048d64", "bwd_preprocess"): (417532416, "7b14b8ee8bec",
                                                     "ncu --set full, one launch"),
    ("c4_causal_b32h16n2048d64", "bwd_dkdv"): (785412864, "7b14b8ee8bec",
                                               "ncu --set full, one launch"),
    ("c4_causal_b32h16n2048d64", "bwd_dq"): (665136384, "7b14b8ee8bec",
                                             "ncu --set full, one launch"),
    ("c5_causal_b2h32n8192d128", "bwd_dkdv"): (782708224, "7b14b8ee8bec",
                                               "ncu --set full, one launch"),
    ("c5_causal_b2h32n8192d128", "bwd_dq"): (665543424, "7b14b8ee8bec",
                                             "ncu --set full, one launch"),
}


# The sources each kernel is compiled from, besides the shared headers: a measured traffic
# figure stays valid while these are unchanged.
COMMON_SOURCES = ("sm100.cuh", "tiles.cuh", "rng.cuh", "launch_impl.cuh", "launch.h")
KERNEL_SOURCES = {
    "fwd": ("fa_fwd.cuh",),
    "bwd_preprocess": ("fa_bwd.cuh",),
    "bwd_dkdv": ("fa_bwd.cuh",),
    "bwd_dq": ("fa_bwd.cuh",),
    "bwd_fused": ("fa_bwd_fused.cuh", "fa_bwd.cuh"),
    "bwd_dq_convert": ("fa_bwd_fused.cuh", "fa_bwd.cuh"),
}


def kernel_source_hash(kernel: str | None = None) -> str:
    """SHA-256 (first 12 hex digits) of the CUDA sources of the library, or, for a kernel
    named in KERNEL_SOURCES, of the shared headers and that kernel's own sources."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_attention_126_b200", "csrc")
    if kernel in KERNEL_SOURCES:
        names = sorted(COMMON_SOURCES + KERNEL_SOURCES[kernel])
    else:
        names = sorted(n for n in os.listdir(csrc) if n.endswith((".cu", ".cuh", ".h")))
    for name in names:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:12]


def measured_traffic(workload: str, kernel: str):
    """(bytes per launch, source) from MEASURED_TRAFFIC if it was taken on the sources the
    kernel is built from now."""
    entry = MEASURED_TRAFFIC.get((workload, kernel))
    if entry is None or entry[1] != kernel_source_hash(kernel):
        return None, None
    return entry[0], entry[2]


def roofline_peak(peaks, region_ms: float):
    """The bf16 peak a kernel timed inside a region of `region_ms` is held to: the burst
    figure (cuBLAS timed alone, full boost clock) for regions under a second, the sustained
    figure (a seconds-long loop under the power cap) for longer ones."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    if region_ms < 1000.0:
        return burst, "burst", sustained
    return sustained, "sustained", sustained


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
def kernel_names(w, fused=False):
    """The kernels of one step, in launch order: the forward, then the backward's delta
    preprocess and either the dK/dV and dQ passes or (fused, head_dim 64) the fused pass and
    the dQ conversion."""
    if not w.backward:
        return ["fwd"]
    if w.d == 64 and fused:
        return ["fwd", "bwd_preprocess", "bwd_fused", "bwd_dq_convert"]
    return ["fwd", "bwd_preprocess", "bwd_dkdv", "bwd_dq"]


def bind_near_gpu(dev_index):
    """Restricts this process to the CPUs next to the GPU (its PCI device's local_cpulist),
    so that pinned host buffers allocated meanwhile live on the GPU's NUMA node; returns the
    previous CPU set to restore, or None when the system does not say (nothing changed)."""
    import torch
    try:
        p = torch.cuda.get_device_properties(dev_index)
        path = "/sys/bus/pci/devices/%04x:%02x:%02x.0/local_cpulist" % (
            p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
        cpus = set()
        for part in open(path).read().strip().split(","):
            lo, _, hi = part.partition("-")
            cpus.update(range(int(lo), int(hi or lo) + 1))
        before = os.sched_getaffinity(0)
        near = before & cpus
        if not near or near == before:
            return None
        os.sched_setaffinity(0, near)
        return before
    except (OSError, ValueError, AttributeError):
        return None


def pack_rows(host, lengths, pin=False):
    """A (B, H, N, d) batch as a packed one: the first lengths[b] rows of entry b, back to
    back, (total, H, d)."""
    import torch
    out = torch.cat([host[b, :, :L].transpose(0, 1) for b, L in enumerate(lengths)], 0)
    out = out.contiguous()
    return out.pin_memory() if pin else out


class Problem:
    """Device buffers of one workload and the library calls of one step.

    A step is the training path: the forward keeps O - bf16(O) (fa_options_t.o_low) and
    the backward's three phases form delta from it; with ALiBi the slopes ride in the same
    options. Each phase is its own C-ABI call, so CUDA events can sit between kernels."""

    def __init__(self, w, dev, host=None, seed=0, plain=False, fused=False):
        import torch
        from exact_attention_126_b200 import fa, workloads
        self.w, self.dev, self.fa = w, dev, fa
        B, H, N, d = w.B, w.H, w.N, w.d
        shape = (B, H, N, d)
        # a packed batch: the sequences back to back as (total, H, d), with cumulative lengths
        self.dims, self.cu, total = None, None, 0
        if w.packed:
            total = sum(w.seq_lengths())
            shape, self.dims = (total, H, d), (B, H, N, d)
        if host is not None:
            # (a packed workload's host inputs are packed already)
            self.q, self.k, self.v, self.do = (host[n].to(dev, non_blocking=True)
                                               for n in ("q", "k", "v", "do"))
        else:
            # i.i.d. N(0, 1) drawn on the device from a seeded generator (timing only: the
            # values' distribution is the workload's, their bits are not the oracle's)
            g = torch.Generator(device=dev)
            g.manual_seed(seed)
            self.q, self.k, self.v, self.do = (
                torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
                .to(torch.bfloat16) for _ in range(4))
        if w.fp8:
            # e4m3 copies of the inputs, descales 1 (N(0, 1) values fit e4m3's range)
            self.q8, self.k8, self.v8 = (t.to(torch.float8_e4m3fn) for t in
                                         (self.q, self.k, self.v))
        self.o = torch.empty_like(self.q)
        self.o_low = torch.empty_like(self.q)
        self.lse = torch.empty((H, total) if w.packed else (B, H, N), dtype=torch.float32,
                               device=dev)
        self.dq, self.dk, self.dv = (torch.empty_like(self.q) for _ in range(3))
        self.slopes = None
        if w.alibi:
            self.slopes = torch.tensor(workloads.alibi_slopes(H), dtype=torch.float32,
                                       device=dev)
        # plain: the forward keeps no residual and delta is formed from the bf16 O
        self.lengths = None
        if w.packed:
            cum = [0]
            for L in w.seq_lengths():
                cum.append(cum[-1] + L)
            self.cu = torch.tensor(cum, dtype=torch.int32, device=dev)
        elif w.varlen:
            self.lengths = torch.tensor(w.seq_lengths(), dtype=torch.int32, device=dev)
        self.opt = fa.options(alibi_slopes=self.slopes, o_low=None if plain else self.o_low,
                              fused=fused, seq_lengths=self.lengths, cu_seqlens=self.cu,
                              total_tokens=total)
        # the workspace holds the row statistics (and with real lengths, the schedule)
        self.ws = torch.empty(max(1, fa.fa_bwd_workspace_bytes_ex(B, H, N, d, self.opt)),
                              dtype=torch.uint8, device=dev)
        self.names = kernel_names(w, fused)
        self.fused = "bwd_fused" in self.names
        self.launches = len(self.names)

    def step(self, sp, evs=None):
        """One pass of the path on stream handle `sp`; evs: len(self.names) + 1 events,
        recorded between kernels."""
        fa, w = self.fa, self.w
        stream = self.stream
        if evs is not None:
            evs[0].record(stream)
        if w.fp8:
            fa.fa_fwd_fp8(self.q8, self.k8, self.v8, 1.0, 1.0, 1.0, self.o, self.lse,
                          w.softmax_scale, w.causal, w.window, sp)
            if evs is not None:
                evs[1].record(stream)
            return
        fa.fa_fwd_ex(self.q, self.k, self.v, self.o, self.lse, self.opt, w.softmax_scale,
                     w.causal, w.window, sp, dims=self.dims)
        if evs is not None:
            evs[1].record(stream)
        if not w.backward:
            return
        fa.fa_bwd_preprocess(self.o, self.do, self.lse, self.ws, self.opt, sp, dims=self.dims)
        if evs is not None:
            evs[2].record(stream)
        if self.fused:
            fa.fa_bwd_fused(self.q, self.k, self.v, self.do, self.ws, self.dk, self.dv,
                            w.softmax_scale, w.causal, w.window, sp, self.opt)
            if evs is not None:
                evs[3].record(stream)
            fa.fa_bwd_dq_convert(self.ws, self.dq, w.softmax_scale, sp)
        else:
            fa.fa_bwd_dkdv(self.q, self.k, self.v, self.do, self.ws, self.dk, self.dv,
                           w.softmax_scale, w.causal, w.window, sp, self.opt, dims=self.dims)
            if evs is not None:
                evs[3].record(stream)
            fa.fa_bwd_dq(self.q, self.k, self.v, self.do, self.ws, self.dq, w.softmax_scale,
                         w.causal, w.window, sp, self.opt, dims=self.dims)
        if evs is not None:
            evs[4].record(stream)

    def time(self, steps, warmup, stream, clocks=None):
        """Device time of `steps` steps after `warmup` untimed ones: (ms per step, per-kernel
        ms per step, bracket ms). L2 is flushed before every step when the inputs fit in it."""
        import torch
        self.stream = stream
        sp = stream.cuda_stream
        w = self.w
        flush = None
        if 4 * w.tensor_bytes() <= L2_BYTES:
            flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=self.dev)
        self.flushed = flush is not None
        for _ in range(warmup):
            if flush is not None:
                flush.zero_()
            self.step(sp)
        torch.cuda.synchronize(self.dev)
        if self.fa.fa_debug_status(sp) != 0:
            raise RuntimeError("a kernel abandoned a bounded wait during warm-up")
        n_ev = len(self.names) + 1
        events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
                  for _ in range(steps)]
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(self.dev)
        t0.record(stream)
        for s in range(steps):
            if flush is not None:
                flush.zero_()
            self.step(sp, events[s])
        t1.record(stream)
        torch.cuda.synchronize(self.dev)
        if self.fa.fa_debug_status(sp) != 0:
            raise RuntimeError("a kernel abandoned a bounded wait in the timed region")
        names = self.names
        per_kernel = {n: 0.0 for n in names}
        step_ms = 0.0
        for evs in events:
            step_ms += evs[0].elapsed_time(evs[-1])
            for i, n in enumerate(names):
                per_kernel[n] += evs[i].elapsed_time(evs[i + 1])
        bracket = t0.elapsed_time(t1)
        ms = step_ms / steps if flush is not None else bracket / steps
        return ms, {n: t / steps for n, t in per_kernel.items()}, bracket


def kernel_flops(w):
    """Algorithmic flops credited to each kernel (the metric's convention): forward = the
    forward count; dK/dV = 2x (S^T, dP^T, dV, dK products); dQ = 0.5x (its dQ product;
    the recomputation of S and dP is not credited); the fused pass = 2.5x (all five
    products); preprocess and dQ conversion move bytes only."""
    f = w.fwd_flops()
    return {"fwd": f, "bwd_preprocess": 0.0, "bwd_dkdv": 2.0 * f, "bwd_dq": 0.5 * f,
            "bwd_fused": 2.5 * f, "bwd_dq_convert": 0.0}


def workload_line(w, ms, per_kernel, flushed):
    """The summary of one workload's timing: ms, TFLOP/s, and the shares of its kernels."""
    value = w.step_flops() / (ms * 1e-3) / 1e12
    kf = kernel_flops(w)
    kernels = {}
    for n, t in per_kernel.items():
        kernels[n] = {"ms": round(t, 5), "share": round(t / sum(per_kernel.values()), 4),
                      "algorithmic_tflops": round(kf[n] / (t * 1e-3) / 1e12, 2) if kf[n] else None}
    line = {"workload": w.name, "pass": "fwd+bwd" if w.backward else "fwd",
            "ms_per_step": round(ms, 5), "tflops": round(value, 2),
            "pct_of_dense_peak": round(100 * value / DATASHEET_BF16_TFLOPS, 2),
            "step_gflop": round(w.step_flops() / 1e9, 3), "kernels": kernels,
            "l2": "L2 flushed before every timed step" if flushed else "inputs larger than L2"}
    if w.window != (-1, -1) and w.window[0] >= 0 and not w.varlen:
        # a sliding window's work is its visible pairs; the causal-halved count that a
        # plain causal problem of this shape would be credited with, for comparison only
        halved = 4.0 * w.B * w.H * w.N * w.N * w.d / 2 * (3.5 if w.backward else 1.0)
        line["tflops_if_counted_causal_halved"] = round(halved / (ms * 1e-3) / 1e12, 2)
        line["causal_halved_overcount"] = round(halved / w.step_flops(), 2)
    if not w.backward:
        # forward-only (launch-bound small) workloads: also microseconds and the compulsory
        # HBM bytes per second
        line["us_per_step"] = round(ms * 1e3, 2)
        line["hbm_gbs_compulsory"] = round(w.fwd_bytes() / (ms * 1e-3) / 1e9, 1)
    return line


def run_ours(args, w, rank, world, local_rank):
    import torch

    from exact_attention_126_b200 import build, fa, synth
    from exact_attention_126_b200.workloads import WORKLOADS

    build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    # the pinned host buffers of the end-to-end run go on the GPU's NUMA node (the process
    # runs on the CPUs next to the GPU while they are allocated)
    cpus_before = bind_near_gpu(local_rank)
    inp_host = synth.attention_inputs(w.B, w.H, w.N, w.d, w.seed_index, with_grad=True,
                                      pin=not w.packed)
    if w.packed:
        inp_host = {n: pack_rows(t, w.seq_lengths(), pin=True) for n, t in inp_host.items()}
    prob = Problem(w, dev, host=inp_host, plain=args.plain, fused=args.fused)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream

    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clocks:
        ms_per_step, per_kernel, bracket_ms = prob.time(args.steps, args.warmup, stream)
    if dist is not None:
        dist.barrier()
        ms_per_step = max_over_ranks(ms_per_step, dist, dev)

    # ---------------------------------------------------------------- end to end
    # The public call a user makes (attention_forward / attention_backward: the same
    # training path, with their own output allocations), inputs copied from pinned host
    # memory and every output read back, each step.
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    q, k, v, do = prob.q, prob.k, prob.v, prob.do
    host_out = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                for n, t in (("o", prob.o), ("lse", prob.lse), ("dq", prob.dq),
                             ("dk", prob.dk), ("dv", prob.dv))}
    in_names = ("q", "k", "v", "do") if w.backward else ("q", "k", "v")
    out_names = ("o", "lse", "dq", "dk", "dv") if w.backward else ("o", "lse")
    if w.fp8:
        # the e4m3 forward's inputs are e4m3 on the host too
        inp_host = {n: inp_host[n].to(torch.float8_e4m3fn).pin_memory() for n in in_names}
        q, k, v = prob.q8, prob.k8, prob.v8
    h2d_bytes = sum(inp_host[n].numel() * inp_host[n].element_size() for n in in_names)
    d2h_bytes = sum(host_out[n].numel() * host_out[n].element_size() for n in out_names)

    # Steps are pipelined over three streams: the host-to-device copies of step k + 1 and
    # the device-to-host copies of step k - 1 run on the two copy engines while step k
    # computes. Inputs go through two device buffer sets, each reused once the step that
    # read it has finished; outputs are fresh tensors from the public calls, kept alive for
    # their copy stream.
    if cpus_before is not None:
        os.sched_setaffinity(0, cpus_before)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    dev_in = [{n: torch.empty_like(t) for n, t in zip(("q", "k", "v", "do"), (q, k, v, do))}
              for _ in range(2)]
    freed = [None, None]  # event: the compute that last read buffer set b has finished

    def e2e_step(step):
        b = step % 2
        bufs = dev_in[b]
        with torch.cuda.stream(s_in):
            if freed[b] is not None:
                s_in.wait_event(freed[b])
            for n in in_names:
                bufs[n].copy_(inp_host[n], non_blocking=True)
            loaded = torch.cuda.Event()
            loaded.record(s_in)
        stream.wait_event(loaded)
        with torch.cuda.stream(stream):  # the outputs are allocated for the compute stream
            if w.fp8:
                res = fa.attention_forward_fp8(bufs["q"], bufs["k"], bufs["v"],
                                               scale=w.softmax_scale, causal=w.causal,
                                               window=w.window, stream=sp)
            else:
                res = fa.attention_forward(bufs["q"], bufs["k"], bufs["v"], w.softmax_scale,
                                           w.causal, w.window, sp, alibi_slopes=prob.slopes,
                                           keep_residual=w.backward, seq_lengths=prob.lengths,
                                           cu_seqlens=prob.cu,
                                           max_seqlen=w.N if w.packed else None)
            outs = [("o", res[0]), ("lse", res[1])]
            if w.backward:
                grads = fa.attention_backward(bufs["q"], bufs["k"], bufs["v"], res[0], res[1],
                                              bufs["do"], w.softmax_scale, w.causal, w.window,
                                              sp, alibi_slopes=prob.slopes, o_low=res[2],
                                              fused=args.fused, seq_lengths=prob.lengths,
                                              cu_seqlens=prob.cu,
                                              max_seqlen=w.N if w.packed else None)
                outs += list(zip(("dq", "dk", "dv"), grads))
            done = torch.cuda.Event()
            done.record(stream)
        freed[b] = done
        with torch.cuda.stream(s_out):
            s_out.wait_event(done)
            for n, t in outs:
                t.record_stream(s_out)
                host_out[n].copy_(t, non_blocking=True)
        return s_out

    e2e_step(0)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(e2e_steps):
        last = e2e_step(i + 1)
    e1.record(last)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if dist is not None:
        e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    del prob

    # ---------------------------------------------------------------- other workloads
    # The other configurations at full size (rank 0 only, after the headline and its
    # end-to-end run; each its own warm-up and timed steps).
    others = {}
    if rank == 0 and not args.no_workloads:
        for name in args.also:
            if WORKLOADS[name].name == w.name:
                continue
            ow = WORKLOADS[name]
            op = Problem(ow, dev, seed=1000 + ow.seed_index, plain=args.plain,
                         fused=args.fused)
            with ClockSampler(local_rank) as oc:
                oms, oker, _ = op.time(max(20, args.steps), args.warmup, stream)
            line = workload_line(ow, oms, oker, op.flushed)
            # the same rate against the measured (else fallback) burst bf16 peak
            pk, pk_src = load_peaks()
            line["pct_of_measured_peak"] = round(
                100 * line["tflops"] / float(pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])), 2)
            line["peak_source"] = pk_src
            line["clocks"] = oc.summary()
            line["data"] = "synthetic (seeded torch.randn on the device, bf16)"
            others[name] = line
            del op
            torch.cuda.empty_cache()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()

    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    flops = w.step_flops()
    value = job_tflops(flops, world, ms_per_step)
    summary = workload_line(w, ms_per_step, per_kernel, prob_flushed(w))
    kernels = summary["kernels"]
    names = list(per_kernel)
    dominant = max(names, key=lambda n: per_kernel[n])
    dom_ms = per_kernel[dominant]
    kf = kernel_flops(w)
    peak, peak_kind, sustained = roofline_peak(peaks, bracket_ms)
    traffic, traffic_src = measured_traffic(w.name, dominant)
    if kf[dominant] > 0:
        achieved = kf[dominant] / (dom_ms * 1e-3) / 1e12
        roofline = {"kernel": dominant, "bound": "tensor", "achieved": round(achieved, 2),
                    "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                    "peak_kind": "bf16 %s (%s): timed region %.0f ms" % (peak_kind, peak_src,
                                                                          bracket_ms),
                    "frac_of_sustained": round(achieved / sustained, 4),
                    "frac_of_datasheet": round(achieved / DATASHEET_BF16_TFLOPS, 4),
                    "traffic": traffic, "traffic_source": traffic_src}
    else:
        nbytes = w.bwd_bytes() if dominant.startswith("bwd") else w.fwd_bytes()
        achieved = nbytes / (dom_ms * 1e-3) / 1e9
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        roofline = {"kernel": dominant, "bound": "hbm", "achieved": round(achieved, 1),
                    "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                    "traffic": traffic, "traffic_source": traffic_src}
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
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
            "workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            "window": list(w.window), "alibi": w.alibi, "varlen": w.varlen, "fp8": w.fp8,
            "pass": "fwd+bwd" if w.backward else "fwd",
            "path": ("plain: delta from the bf16 O" if args.plain else
                     "training path: forward keeps O - bf16(O) for the backward's delta")
                    + ("; fused backward (dQ by fp32 bulk reductions)" if args.fused else ""),
            "kernels": list(per_kernel),
            "step_gflop": round(flops / 1e9, 3),
            "parallelism": "replicas" if world > 1 else "single",
            "l2": summary["l2"],
        },
        "pct_of_dense_peak": round(100 * value / world / DATASHEET_BF16_TFLOPS, 2),
        "pct_of_measured_peak": round(100 * value / world / burst, 2),
        "clocks": clocks.summary(),
        "e2e": {"value": round(job_tflops(flops, world, e2e_ms), 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 3), "steps": e2e_steps,
                "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
                "host_buffers": "pinned, on the GPU's NUMA node" if cpus_before is not None
                else "pinned (the CPU affinity was left as it was)"},
        "gpu_launches": len(per_kernel) * args.steps,
        "kernels": kernels,
        "roofline": roofline,
        "kernel_source_hash": kernel_source_hash(),
    }
    if others:
        line["workloads"] = others
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    return line


def prob_flushed(w) -> bool:
    return 4 * w.tensor_bytes() <= L2_BYTES


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


def _oracle_head(orc, w, b, h):
    """Runs the oracle, as it stands, on the (batch b, head h) problem of the workload;
    returns (seconds, the problem's flops by the metric's convention)."""
    x = _oracle_sample(w, b, h)
    slope = _head_slope(w, h)
    lengths = [w.seq_lengths()[b]] if w.varlen else None
    pairs = w.visible_pairs(lengths[0]) if w.varlen else None
    flops = (4.0 * w.d * pairs * (3.5 if w.backward else 1.0) if w.varlen
             else w.step_flops() / (w.B * w.H))
    t0 = time.perf_counter()
    orc.fwd(x["q"], x["k"], x["v"], w.softmax_scale, w.causal, w.window, slope,
            lengths=lengths)
    if w.backward:
        orc.bwd(x["q"], x["k"], x["v"], x["do"], w.softmax_scale, w.causal, w.window, slope,
                lengths=lengths)
    return time.perf_counter() - t0, flops


def cpu_baseline(w, seconds: float):
    """Times the fp64 oracle, as it stands, on whole (batch, head) problems of the workload
    until `seconds` have passed (at least one head)."""
    import oracle
    orc = oracle.default()
    done, elapsed, flops = 0, 0.0, 0.0
    BH = w.B * w.H
    while elapsed < seconds and done < BH:
        b, h = divmod(done, w.H)
        dt, f = _oracle_head(orc, w, b, h)
        elapsed += dt
        flops += f
        done += 1
    return {"value": round(flops / elapsed / 1e12, 6), "unit": "TFLOP/s",
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
    heads_per_step = 1

    def one(idx):
        b, h = divmod(idx % BH, w.H)
        return _oracle_head(orc, w, b, h)

    for i in range(args.warmup):
        one(i)
    runs = [one(args.warmup + s) for s in range(args.steps)]
    total = sum(t for t, _ in runs)
    ms_per_step = total * 1e3 / args.steps
    value = sum(f for _, f in runs) / total / 1e12
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
    ap.add_argument("--workload", default="c4",
                    help="c1, c2, c3, c4, c5c, c5w, c4a, c4v, c4p or c5f8")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--also", default="c2,c3,c4,c5c,c5w,c4v,c4p,c5f8",
                    help="other workloads timed at full size in the same run (comma list)")
    ap.add_argument("--fused", action="store_true",
                    help="time the fused backward (dQ by fp32 bulk reductions) at head_dim 64")
    ap.add_argument("--plain", action="store_true",
                    help="time the path without the O residual (delta from the bf16 O)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time the headline workload only")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    args.also = [x for x in args.also.split(",") if x]

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
