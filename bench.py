#!/usr/bin/env python
"""Throughput of the element-wise recurrence scans on B200, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl b200|reference] [--no-rows]

A step is one minGRU scan (activations, the scan over T, store) over one
batch of the workload, with inputs resident in HBM.  The default workload is
the largest single-GPU configuration, the minGRU scan with carried state
B=16 T=2048 D=4096 with bf16 inputs and output and fp32 arithmetic (k, hx ~
N(0,1), h0 ~ U(0.1,1)).  Its inputs (537 MB) and output (268 MB) are larger
than the 126 MB L2, so back-to-back steps do not hit in L2.

Metric: scan HBM GB/s = algorithmic bytes (inputs read once + output written
once + initial state) per step / time per step, summed over GPUs.  Also
reported: Gelem/s, the dominant kernel's roofline fraction against the
measured HBM copy bandwidth, the end-to-end figure through the public API
with the inputs in pinned host memory (host<->device copies timed), the CPU
oracle on a bounded sample of the same workload, and one line per other hot
path row (MinMax scan, long sequence, bf16 I/O, small shape, decode step).

Multi-GPU (torchrun): every rank scans its own batch shard of the same size
(weak scaling); channels are independent, so there is no data-path
collective.  Timing is the max over ranks of device-measured time.

--impl reference times the CPU oracle (the reference arm of this method) on
the host cores, on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from scan_gated_rnns_b200.synth import BENCH_WORKLOAD, WORKLOADS, generate  # noqa: E402

METRIC = "scan HBM GB/s (fraction of B200 peak) and Gelem/s at BxTxD, vs CPU oracle"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
# the device sources of each profiled kernel: a committed ncu summary's DRAM
# traffic is reported only while these are unchanged since its capture
_ENGINE = "scan_gated_rnns_b200/csrc/scan_engine.cuh"
KERNEL_SOURCES = {
    "scan_kernel": [_ENGINE],
    "scan_sequential_kernel": [_ENGINE, "scan_gated_rnns_b200/csrc/scan_sequential.cuh"],
    "scan_sequential_pair_kernel": [_ENGINE, "scan_gated_rnns_b200/csrc/scan_sequential.cuh"],
    "scan_sequential_pair2_kernel": [_ENGINE, "scan_gated_rnns_b200/csrc/scan_sequential.cuh"],
    "scan_sequential_backward_kernel": [_ENGINE, "scan_gated_rnns_b200/csrc/scan_backward.cuh",
                                        "scan_gated_rnns_b200/csrc/scan_sequential.cuh"],
    "scan_backward_kernel": [_ENGINE, "scan_gated_rnns_b200/csrc/scan_backward.cuh"],
    "scan_pipelined_backward_kernel": [_ENGINE, "scan_gated_rnns_b200/csrc/scan_backward.cuh",
                                       "scan_gated_rnns_b200/csrc/scan_pipelined_backward.cuh"],
    "mingru_projected_scan_kernel": [_ENGINE, "scan_gated_rnns_b200/csrc/projected_scan.cuh"],
}


# ------------------------------------------------------------------ helpers

def kernel_source_sha(kernel: str = "scan_kernel") -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured (MEASURED_PEAKS.json hbm_gbs, copy bandwidth)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s earlier pool measurement)"


def recorded_traffic(workload: str, kernel: str = "scan_kernel"):
    """dram bytes per launch from the committed ncu summary of this kernel and
    workload, if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.startswith("- "):
                k, v = line[2:].split(":", 1)
                v = v.strip()
                fields[k.strip()] = v[1:].split("`", 1)[0] if v.startswith("`") else v
    if fields.get("kernel_source_sha") != kernel_source_sha(kernel):
        return None
    try:
        return int(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """SM clock, power and clock-event reasons via NVML, polled from a thread
    every `period` seconds; samples are kept with host timestamps so the ones
    inside the timed window can be selected."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index: int, period: float = 0.002):
        self.samples = []
        self.period = period
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            self.nv = pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            handle = None
            for cand in (uuid, "GPU-" + uuid):
                try:
                    handle = pynvml.nvmlDeviceGetHandleByUUID(cand)
                    break
                except Exception:
                    continue
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.h = handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report the clocks as unknown
            self.err = str(e)

    def _read(self):
        nv = self.nv
        sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        try:
            pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
        except Exception:
            pw = None
        return sm, rs, pw

    def sample_now(self):
        """One sample from the calling thread (see timed_launches)."""
        if not self.ok:
            return
        try:
            sm, rs, pw = self._read()
            self.samples.append((time.time(), sm, rs, pw))
        except Exception:
            pass

    def start(self):
        if not self.ok:
            return self
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    sm, rs, pw = self._read()
                    self.samples.append((time.time(), sm, rs, pw))
                except Exception:
                    pass
                time.sleep(self.period)

        self._t = threading.Thread(target=loop, daemon=True)
        self._t.start()
        return self

    def stop(self):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": "unavailable: " + getattr(self, "err", "")}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        used = inside
        where = "timed region"
        if not inside:   # region shorter than one poll: the nearest samples around it
            used = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
            where = "nearest to the timed region (shorter than the poll period)"
        reasons = set()
        for _, _, rs, _ in used:
            for name, bit in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        sm = [s[1] for s in used]
        pw = [s[3] for s in used if s[3] is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(used), "window": where,
                "power_w_max": max(pw) if pw else None, "source": "nvml"}


# ------------------------------------------------------------ distribution

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def shard_seed(base_seed: int, rank: int) -> int:
    """Each rank scans its own batch shard: same shape, its own seeded draws."""
    return base_seed + 1000 * rank


def reduce_max(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None) -> None:
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate(bytes_per_step: int, elems_per_step: int, steps: int, max_seconds: float, world: int):
    """Whole-job throughput: every rank moved bytes_per_step per step."""
    return {
        "gbs": world * bytes_per_step * steps / max_seconds / 1e9,
        "gelems": world * elems_per_step * steps / max_seconds / 1e9,
        "ms_per_step": max_seconds * 1e3 / steps,
    }


# ---------------------------------------------------------------- GPU timing

# GPU cycles of the spin queued ahead of a device-timed region (~50 us at
# the B200's 1965 MHz boost clock)
LEAD_CYCLES = 100_000


def timed_launches(fn, steps: int, stream, while_busy=None, lead: bool = True):
    """Time `steps` calls of fn with CUDA events on the launching stream: the
    whole region and each launch.  Returns (total_s, mean_launch_s).
    `while_busy`, if given, is called on the host between the last launch
    being queued and the stream reaching its end (the clock sampler reads
    NVML there, so that its samples fall inside the timed region however
    short it is).  lead: a short GPU spin is queued before the start event,
    so that the host has queued the first launches by the time the stream
    reaches it; otherwise, after the synchronize that precedes every timed
    region, the first interval would hold the host's ~20 us of launch
    latency on an idle GPU as well as the kernel (measured: the first of 20
    back-to-back launches 100 us against 76 us for the rest).  Off for the
    end-to-end and per-call timings, whose host work is part of what they
    measure."""
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if lead:
        with torch.cuda.stream(stream):
            torch.cuda._sleep(LEAD_CYCLES)
    t0.record(stream)
    for i in range(steps):
        starts[i].record(stream)
        fn()
        ends[i].record(stream)
    t1.record(stream)
    if while_busy is not None:
        while not t1.query():
            while_busy()
            time.sleep(2e-4)
    torch.cuda.synchronize()
    total = t0.elapsed_time(t1) / 1e3
    per = statistics.mean(s.elapsed_time(e) for s, e in zip(starts, ends)) / 1e3
    return total, per


def scan_fn(w, p, q, init, out, ws):
    import scan_gated_rnns_b200 as sgr
    f = sgr.mingru_scan if w.op == "mingru" else sgr.minmax_scan
    return lambda: f(p, q, init, out=out, workspace=ws)


PASS_SUFFIX = {"backward": "_backward", "decay": "_decay", "decay_backward": "_decay_backward", "log": "_log"}


def plan_kernel(plan) -> str:
    """The device kernel a scan plan launches (the library's kernel kinds)."""
    return {1: "sgr::scan_tile_kernel", 2: "sgr::scan_pipelined_kernel", 3: "sgr::scan_pipelined_kernel",
            4: "sgr::scan_sequential_kernel", 5: "sgr::scan_sequential_kernel (split rows)",
            6: "sgr::scan_sequential_pair_kernel",
            7: "sgr::scan_sequential_pair2_kernel",
            8: "sgr::scan_sequential_pair2_kernel (four warps)"}.get(plan["kernel"], "sgr::scan_kernel")


def profile_kernel(plan) -> str:
    """The name a plan's kernel is filed under in profiles/: the chunked
    kernels as scan_kernel, the channel-sequential ones by their own names."""
    if plan["kernel"] in (4, 5):
        return "sgr::scan_sequential_kernel"
    if plan["kernel"] == 6:
        return "sgr::scan_sequential_pair_kernel"
    if plan["kernel"] in (7, 8):
        return "sgr::scan_sequential_pair2_kernel"
    return "sgr::scan_kernel"


def backward_kernel(w) -> str:
    """The device kernel the gradient of workload w launches."""
    import scan_gated_rnns_b200 as sgr
    kind = sgr._abi.lib().sgr_backward_kernel(0 if w.op == "mingru" else 1, w.B, w.T, w.D,
                                              0 if w.dtype == "f32" else 1, 1)
    return {4: "sgr::scan_sequential_backward_kernel",
            2: "sgr::scan_pipelined_backward_kernel"}.get(kind, "sgr::scan_backward_kernel")


def measure_row(w, device, steps=10, warmup=3):
    """One other hot-path row, timed alone (inputs larger than L2 except the
    small shape, which is launch-latency bound)."""
    import scan_gated_rnns_b200 as sgr
    p, q, init = generate(w, device=device)
    out = torch.empty_like(p)
    ws = sgr.Workspace(sgr.workspace_size(w.op, w.B, w.T, w.D, p.dtype), device)
    fn = scan_fn(w, p, q, init, out, ws)
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)
    total, per = timed_launches(fn, steps, stream)
    bytes_ = w.algorithmic_bytes()
    peak, _ = hbm_peak()
    gbs = bytes_ / per / 1e9
    plan = sgr._abi.plan(0 if w.op == "mingru" else 1, w.B, w.T, w.D,
                         0 if w.dtype == "f32" else 1, True)
    row = {"op": f"{w.op}_scan", "B": w.B, "T": w.T, "D": w.D, "io_dtype": w.dtype,
           "us_per_launch": round(per * 1e6, 2), "gbs": round(gbs, 1),
           "gelem_per_s": round(w.n_elems / per / 1e9, 2), "roofline_frac": round(gbs / peak, 4),
           "bytes_per_launch": bytes_, "kernel": plan_kernel(plan),
           "tile": f"{plan['tile_rows']}x{plan['tile_channels']}", "n_tiles": plan["n_tiles"]}
    if bytes_ < 64 << 20:
        # fits in L2 and is over in microseconds: the host's call overhead shows in
        # the per-call events, so also time the launches replayed from a CUDA graph
        stream = torch.cuda.Stream(device)
        stream.wait_stream(torch.cuda.current_stream(device))
        with torch.cuda.stream(stream):
            fn()
            stream.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                for _ in range(steps):
                    fn()
            graph.replay()
            stream.synchronize()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            graph.replay()
            t1.record(stream)
            stream.synchronize()
        g_per = t0.elapsed_time(t1) / 1e3 / steps
        row["us_per_launch_graph"] = round(g_per * 1e6, 2)
        row["note"] = "fits in L2 (inputs stay cached between launches): latency, not bandwidth"
        del graph
    del p, q, init, out, ws
    return row


def measure_backward_row(w, device, steps=10, warmup=3):
    """Gradient of one scan (dL/d out given): reads the two inputs, the forward
    output and the upstream gradient, writes the two input gradients (and the
    initial state's): 6 (B, T, D) tensors per launch."""
    import scan_gated_rnns_b200 as sgr
    p, q, init = generate(w, device=device)
    fwd = (sgr.mingru_scan if w.op == "mingru" else sgr.minmax_scan)(p, q, init)
    g = torch.Generator(device=device).manual_seed(w.seed + 17)
    gy = torch.randn(p.shape, device=device, generator=g).to(p.dtype)
    op = 0 if w.op == "mingru" else 1
    dt = 0 if w.dtype == "f32" else 1
    ws = sgr.Workspace(sgr._abi.lib().sgr_backward_workspace_size(op, w.B, w.T, w.D, dt), device)
    bwd = sgr.mingru_scan_backward if w.op == "mingru" else sgr.minmax_scan_backward
    fn = lambda: bwd(p, q, init, fwd, gy, init is not None, workspace=ws)  # noqa: E731
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    total, per = timed_launches(fn, steps, torch.cuda.current_stream(device))
    bytes_ = 6 * w.n_elems * w.elem_bytes + (2 * w.B * w.D * w.elem_bytes if init is not None else 0)
    peak, _ = hbm_peak()
    gbs = bytes_ / per / 1e9
    del p, q, init, fwd, gy, ws
    return {"op": f"{w.op}_scan_backward", "B": w.B, "T": w.T, "D": w.D, "io_dtype": w.dtype,
            "us_per_launch": round(per * 1e6, 2), "gbs": round(gbs, 1),
            "gelem_per_s": round(w.n_elems / per / 1e9, 2), "roofline_frac": round(gbs / peak, 4),
            "bytes_per_launch": bytes_, "kernel": backward_kernel(w)}


def measure_decay_rows(w, device, steps=10, warmup=3):
    """minGRU with time decay on workload w: forward and gradient.  Gaps
    delta_t ~ Exp(1) per (b, t), rates lambda ~ U(0, 1) per channel (fp32)."""
    import scan_gated_rnns_b200 as sgr
    p, q, init = generate(w, device=device)
    g = torch.Generator(device=device).manual_seed(w.seed + 29)
    dt = torch.empty(w.B, w.T, device=device).exponential_(1.0, generator=g)
    lam = torch.rand(w.D, device=device, generator=g)
    out = torch.empty_like(p)
    ws = sgr.Workspace(max(sgr.workspace_size("mingru", w.B, w.T, w.D, p.dtype),
                           sgr._abi.lib().sgr_backward_workspace_size(0, w.B, w.T, w.D,
                                                                      0 if w.dtype == "f32" else 1)),
                       device)
    fwd = lambda: sgr.mingru_scan_decay(p, q, init, dt, lam, out=out, workspace=ws)  # noqa: E731
    for _ in range(warmup):
        fwd()
    torch.cuda.synchronize()
    _, per_f = timed_launches(fwd, steps, torch.cuda.current_stream(device))
    gy = torch.randn(p.shape, device=device, generator=g).to(p.dtype)
    bwd = lambda: sgr.mingru_scan_decay_backward(p, q, init, dt, lam, out, gy, workspace=ws)  # noqa: E731
    for _ in range(warmup):
        bwd()
    torch.cuda.synchronize()
    _, per_b = timed_launches(bwd, steps, torch.cuda.current_stream(device))
    peak, _ = hbm_peak()
    extra = w.B * w.T * 4 + w.D * 4                     # gaps and rates
    fb = w.algorithmic_bytes() + extra
    bb = 6 * w.n_elems * w.elem_bytes + extra + w.D * 4 + \
        (2 * w.B * w.D * w.elem_bytes if init is not None else 0)
    del p, q, init, out, ws, gy, dt, lam
    plan = sgr._abi.plan(0, w.B, w.T, w.D, 0 if w.dtype == "f32" else 1, True, decay=True)
    rows = {}
    for kind, per, bytes_, kern in (("", per_f, fb, plan_kernel(plan)),
                                    ("_backward", per_b, bb, backward_kernel(w))):
        gbs = bytes_ / per / 1e9
        rows[w.name.replace("mingru_", f"mingru_decay{kind}_", 1)] = {
            "op": f"mingru_scan_decay{kind}", "B": w.B, "T": w.T, "D": w.D, "io_dtype": w.dtype,
            "us_per_launch": round(per * 1e6, 2), "gbs": round(gbs, 1),
            "gelem_per_s": round(w.n_elems / per / 1e9, 2), "roofline_frac": round(gbs / peak, 4),
            "bytes_per_launch": bytes_, "kernel": kern}
    return rows


def measure_log_row(w, device, steps=10, warmup=3):
    """The minGRU scan evaluated in log space (mingru_scan_log) beside the
    linear pairs on the same inputs: once with the linear scan's own plan and
    once forced onto the chunked kernel the log-space scan runs, so that the
    two times differ only in the evaluation domain."""
    import scan_gated_rnns_b200 as sgr
    p, q, init = generate(w, device=device)
    out = torch.empty_like(p)
    ws = sgr.Workspace(max(sgr.workspace_size("mingru_log", w.B, w.T, w.D, p.dtype),
                           sgr.workspace_size("mingru", w.B, w.T, w.D, p.dtype)), device)
    dt = 0 if w.dtype == "f32" else 1
    plan = sgr._abi.plan(sgr._abi.SGR_OP_MINGRU_LOG, w.B, w.T, w.D, dt)
    stream = torch.cuda.current_stream(device)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        return timed_launches(fn, steps, stream)[1]

    per_log = timed(lambda: sgr.mingru_scan_log(p, q, init, out=out, workspace=ws))
    per_lin = timed(lambda: sgr.mingru_scan(p, q, init, out=out, workspace=ws))
    sgr.set_kernel_override(plan["kernel"])
    try:
        per_same = timed(lambda: sgr.mingru_scan(p, q, init, out=out, workspace=ws))
    finally:
        sgr.set_kernel_override(0)
    lin_plan = sgr._abi.plan(0, w.B, w.T, w.D, dt)
    bytes_ = w.algorithmic_bytes()
    peak, _ = hbm_peak()
    gbs = bytes_ / per_log / 1e9
    del p, q, init, out, ws
    return {"op": "mingru_scan_log", "B": w.B, "T": w.T, "D": w.D, "io_dtype": w.dtype,
            "us_per_launch": round(per_log * 1e6, 2), "gbs": round(gbs, 1),
            "gelem_per_s": round(w.n_elems / per_log / 1e9, 2), "roofline_frac": round(gbs / peak, 4),
            "bytes_per_launch": bytes_, "kernel": plan_kernel(plan) + " (log-space pairs)",
            "linear_same_kernel_us": round(per_same * 1e6, 2),
            "linear_us": round(per_lin * 1e6, 2), "linear_kernel": plan_kernel(lin_plan)}


def measure_summary_row(w, device, steps=10, warmup=3):
    """The slice summary of the split-time-axis path (the extra pass a rank
    makes before the exchange): reads both inputs once."""
    from scan_gated_rnns_b200 import sharded
    p, q, _ = generate(w, device=device)
    fn = lambda: sharded.scan_summary(w.op, p, q)   # noqa: E731
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    _, per = timed_launches(fn, steps, torch.cuda.current_stream(device))
    bytes_ = 2 * w.n_elems * w.elem_bytes + w.B * w.D * 8
    peak, _ = hbm_peak()
    gbs = bytes_ / per / 1e9
    del p, q
    return {"op": f"{w.op}_scan_summary", "B": w.B, "T": w.T, "D": w.D, "io_dtype": w.dtype,
            "us_per_call": round(per * 1e6, 2), "gbs": round(gbs, 1), "roofline_frac": round(gbs / peak, 4),
            "bytes_per_call": bytes_, "kernel": "sgr::scan_summary_kernel + fold_partials_kernel"}


def bf16_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
    except Exception:
        return 1590.0, "fallback (1.59 PFLOP/s earlier pool measurement)"


PROJ_TILE = (256, 64)     # tokens x channels per tile of the fused kernel
PROJECTED = {"B": 8, "T": 4096, "D": 1024, "d_in": 1024}


def projected_inputs(device, B, T, D, d_in, seed=31):
    g = torch.Generator(device=device).manual_seed(seed)
    x = torch.randn(B, T, d_in, device=device, generator=g).to(torch.bfloat16)
    w = (torch.randn(2 * D, d_in, device=device, generator=g) / d_in ** 0.5).to(torch.bfloat16)
    h0 = torch.rand(B, D, device=device, generator=g) * 0.9 + 0.1
    return x, w, h0


def measure_projected_row(device, steps=10, warmup=3, B=8, T=4096, D=1024, d_in=1024):
    """The minGRU layer's input projection fused with the scan (tensor cores),
    against the same work unfused: two cuBLAS bf16 GEMMs writing k and hx,
    then the bf16 scan."""
    import scan_gated_rnns_b200 as sgr
    x, w, h0 = projected_inputs(device, B, T, D, d_in)
    out = torch.empty(B, T, D, device=device)
    ws = sgr.Workspace(sgr._abi.lib().sgr_projected_workspace_size(B, T, D), device)
    fused = lambda: sgr.mingru_projected_scan(x, w, h0, out=out, workspace=ws)  # noqa: E731
    for _ in range(warmup):
        fused()
    torch.cuda.synchronize()
    _, per = timed_launches(fused, steps, torch.cuda.current_stream(device))
    k = torch.empty(B, T, D, device=device, dtype=torch.bfloat16)
    hx = torch.empty_like(k)
    hb = torch.empty_like(k)
    wsb = sgr.Workspace(sgr.workspace_size("mingru", B, T, D, torch.bfloat16), device)
    h0b = h0.to(torch.bfloat16)
    wk, wh = w[:D], w[D:]

    def unfused():
        torch.matmul(x, wk.t(), out=k)
        torch.matmul(x, wh.t(), out=hx)
        sgr.mingru_scan(k, hx, h0b, out=hb, workspace=wsb)

    for _ in range(warmup):
        unfused()
    torch.cuda.synchronize()
    _, per_u = timed_launches(unfused, steps, torch.cuda.current_stream(device))
    flops = 2.0 * B * T * d_in * 2 * D
    peak, src = bf16_peak()
    del x, w, h0, out, ws, k, hx, hb, wsb
    return {"op": "mingru_projected_scan", "B": B, "T": T, "D": D, "d_in": d_in, "io_dtype": "bf16 in, f32 out",
            "us_per_launch": round(per * 1e6, 2), "tflops": round(flops / per / 1e12, 1),
            "roofline_frac": round(flops / per / 1e12 / peak, 4), "peak_tflops": peak, "peak_source": src,
            "flops_per_launch": flops, "kernel": "sgr::mingru_projected_scan_kernel (tcgen05)",
            "unfused_us": round(per_u * 1e6, 2),
            "unfused": "torch.matmul bf16 x2 (cuBLAS) to k, hx + mingru_scan bf16"}


def measure_step_row(device, B=8, D=1024, calls=200, warmup=10):
    """Decode step on (B, D): latency-bound; microseconds per call."""
    import scan_gated_rnns_b200 as sgr
    g = torch.Generator(device=device).manual_seed(77)
    k = torch.randn(B, D, device=device, generator=g)
    hx = torch.randn(B, D, device=device, generator=g)
    h = torch.rand(B, D, device=device, generator=g) + 0.1
    fn = lambda: sgr.mingru_step(k, hx, h, out=h)   # noqa: E731
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    total, per = timed_launches(fn, calls, torch.cuda.current_stream(device), lead=False)
    # the same steps replayed from a CUDA graph: the device-side time of one
    # step without the host's per-call overhead (token-by-token decoding
    # captures its step loop the same way)
    stream = torch.cuda.Stream(device)
    stream.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(stream):
        fn()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for _ in range(calls):
                fn()
        graph.replay()
        stream.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        graph.replay()
        t1.record(stream)
        stream.synchronize()
    g_per = t0.elapsed_time(t1) / 1e3 / calls
    del graph
    row = {"op": "mingru_step", "B": B, "D": D, "io_dtype": "f32",
           "us_per_call": round(total / calls * 1e6, 2),
           "us_per_launch_event": round(per * 1e6, 2),
           "us_per_step_graph": round(g_per * 1e6, 2), "bytes_per_call": 4 * 4 * B * D}
    row["c_host_loop"] = step_host_loop(device, B, D)
    return row


def step_host_loop(device, B, D, steps=2000, warmup=100):
    """The same decode step called from a plain C++ host loop through the C
    ABI (scan_gated_rnns_b200/step_latency, built with the library): the
    per-token cost without Python.  Its own process on the same device."""
    from scan_gated_rnns_b200 import build as sgr_build
    exe = sgr_build.STEP_EXE
    if not os.path.exists(exe):
        return {"unavailable": "step_latency not built"}
    env = dict(os.environ)
    idx = device.index if device.index is not None else 0
    vis = env.get("CUDA_VISIBLE_DEVICES")
    if vis:
        env["CUDA_VISIBLE_DEVICES"] = vis.split(",")[idx]
    else:
        env["CUDA_VISIBLE_DEVICES"] = str(idx)
    try:
        out = subprocess.run([exe, str(B), str(D), str(steps), str(warmup)], env=env, capture_output=True,
                             text=True, timeout=120)
    except (OSError, subprocess.TimeoutExpired) as e:
        return {"unavailable": f"step_latency did not run: {e}"}
    if out.returncode != 0:
        return {"unavailable": (out.stderr or out.stdout).strip()[-200:]}
    return json.loads(out.stdout.strip().splitlines()[-1])


def usable_cores() -> int:
    """CPUs this process may run on (its affinity mask where the platform has
    one, else the logical CPU count), capped at 32 threads."""
    try:
        n = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        n = os.cpu_count() or 1
    return max(1, min(n, 32))


def cpu_baseline(w, p, q, init, budget_s: float = 12.0, cpu_target_s: float = 12.0):
    """The fp64 CPU oracle as it stands, on a bounded sample of the workload:
    whole batch rows (all T and D of each), threads over rows."""
    import oracle
    cores = usable_cores()
    row = w.T * w.D
    # time one row first, then size the sample to about `budget_s` of wall time
    p1, q1 = p[:1].cpu(), q[:1].cpu()
    i1 = init[:1].cpu() if init is not None else None
    t = time.perf_counter()
    oracle.mingru_linear(p1, q1, i1) if w.op == "mingru" else oracle.minmax(p1, q1, i1)
    one = time.perf_counter() - t
    rows = int(max(1, min(w.B, budget_s / max(one, 1e-6) * min(cores, w.B))))
    threads = min(cores, rows)
    ps, qs = p[:rows].cpu(), q[:rows].cpu()
    ins = init[:rows].cpu() if init is not None else None
    fn = oracle.mingru_linear if w.op == "mingru" else oracle.minmax
    t = time.perf_counter()
    fn(ps, qs, ins, threads=threads)
    wall = time.perf_counter() - t
    # when the whole sample (every batch row) is over in well under
    # `cpu_target_s` core-seconds, repeat the pass so the rate rests on about
    # that much CPU work (at most 50 passes)
    passes = int(min(50, max(1, math.ceil(cpu_target_s / max(wall * threads, 1e-6)))))
    for _ in range(passes - 1):
        t0 = time.perf_counter()
        fn(ps, qs, ins, threads=threads)
        wall += time.perf_counter() - t0
    bytes_ = (3 * rows * row * w.elem_bytes + (rows * w.D * w.elem_bytes if init is not None else 0)) * passes
    # the first pass over one batch row ran on one thread: the single-core rate
    one_bytes = 3 * row * w.elem_bytes + (w.D * w.elem_bytes if init is not None else 0)
    single = {"value": round(one_bytes / max(one, 1e-9) / 1e9, 4), "unit": UNIT,
              "gelem_per_s": round(row / max(one, 1e-9) / 1e9, 5), "seconds": round(one, 3),
              "sample": f"batch row 0 ({w.T}x{w.D} elements), 1 thread, one pass"}
    return {"value": round(bytes_ / wall / 1e9, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
            "single_thread": single,
            "gelem_per_s": round(passes * rows * row / wall / 1e9, 5), "seconds": round(wall, 2),
            "cpu_seconds": round(wall * threads, 1), "passes": passes,
            "sample": f"batch rows 0..{rows - 1} of the workload ({rows}x{w.T}x{w.D} elements), "
                      f"{passes} pass(es), fp64 {'linear-space minGRU' if w.op == 'mingru' else 'MinMax'} "
                      f"oracle, {threads} thread(s) over rows; host has {os.cpu_count()} logical CPUs, "
                      f"{usable_cores()} usable by this process (affinity mask, capped at 32)"}


# ------------------------------------------------------------------- arms

def run_b200(args):
    import scan_gated_rnns_b200 as sgr
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the scans have no CPU path)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    w = WORKLOADS[args.workload]
    p, q, init = generate(w, seed=shard_seed(w.seed, rank), device=device)
    out = torch.empty_like(p)
    ws = sgr.Workspace(sgr.workspace_size(w.op, w.B, w.T, w.D, p.dtype), device)
    fn = scan_fn(w, p, q, init, out, ws)
    stream = torch.cuda.current_stream(device)
    bytes_step = w.algorithmic_bytes()
    # the chunked kernels' profiles are filed as scan_kernel; the channel-
    # sequential kernels (wide batches) under their own names
    kernel_name = profile_kernel(sgr._abi.plan(0 if w.op == "mingru" else 1, w.B, w.T, w.D,
                                               0 if w.dtype == "f32" else 1, True))
    if args.pass_ == "projected":
        # the input projection fused with the scan: x (B, T, d_in) and W (2 D, d_in) bf16
        P = PROJECTED
        x, wproj, hp0 = projected_inputs(device, P["B"], P["T"], P["D"], P["d_in"], seed=shard_seed(31, rank))
        hout = torch.empty(P["B"], P["T"], P["D"], device=device)
        wsp = sgr.Workspace(sgr._abi.lib().sgr_projected_workspace_size(P["B"], P["T"], P["D"]), device)
        fn = lambda: sgr.mingru_projected_scan(x, wproj, hp0, out=hout, workspace=wsp)  # noqa: E731
        bytes_step = 2 * P["B"] * P["T"] * P["d_in"] + 4 * P["D"] * P["d_in"] + 4 * P["B"] * P["T"] * P["D"]
        kernel_name = "sgr::mingru_projected_scan_kernel"
        ws = wsp
        args.no_e2e = True
    if args.pass_ == "backward":
        # the gradient of the same scan: reads both inputs, the forward output
        # and dL/d out, writes both input gradients (and the initial state's)
        fn()
        g = torch.Generator(device=device).manual_seed(w.seed + 17)
        gy = torch.randn(p.shape, device=device, generator=g).to(p.dtype)
        wsb = sgr.Workspace(sgr._abi.lib().sgr_backward_workspace_size(
            0 if w.op == "mingru" else 1, w.B, w.T, w.D, 0 if w.dtype == "f32" else 1), device)
        bwd = sgr.mingru_scan_backward if w.op == "mingru" else sgr.minmax_scan_backward
        fn = lambda: bwd(p, q, init, out, gy, init is not None, workspace=wsb)  # noqa: E731
        bytes_step = 6 * w.n_elems * w.elem_bytes + (2 * w.B * w.D * w.elem_bytes if init is not None else 0)
        kernel_name = backward_kernel(w)
        ws = wsb
        args.no_e2e = True
    profile_key = w.name
    if args.pass_ == "log":
        # the same scan evaluated in log space (mingru_scan_log), for the
        # comparison of evaluation domains
        if w.op != "mingru":
            raise SystemExit("bench.py: the log-space evaluation is a minGRU form")
        wsl = sgr.Workspace(sgr.workspace_size("mingru_log", w.B, w.T, w.D, p.dtype), device)
        fn = lambda: sgr.mingru_scan_log(p, q, init, out=out, workspace=wsl)  # noqa: E731
        kernel_name = plan_kernel(sgr._abi.plan(sgr._abi.SGR_OP_MINGRU_LOG, w.B, w.T, w.D,
                                                0 if w.dtype == "f32" else 1, True))
        kernel_name = "sgr::scan_kernel" if "sequential" not in kernel_name else kernel_name
        profile_key = w.name.replace("mingru_", "mingru_log_", 1)
        ws = wsl
        args.no_e2e = True
    if args.pass_ in ("decay", "decay_backward"):
        # the time-decayed minGRU on the workload: gaps ~ Exp(1) per (b, t),
        # rates ~ U(0, 1) per channel, fp32 (the decay rows' recipe)
        if w.op != "mingru":
            raise SystemExit("bench.py: time decay is a minGRU variant")
        g = torch.Generator(device=device).manual_seed(w.seed + 29)
        gaps = torch.empty(w.B, w.T, device=device).exponential_(1.0, generator=g)
        lam = torch.rand(w.D, device=device, generator=g)
        code = 0 if w.dtype == "f32" else 1
        wsd = sgr.Workspace(max(sgr.workspace_size("mingru", w.B, w.T, w.D, p.dtype),
                                sgr._abi.lib().sgr_backward_workspace_size(0, w.B, w.T, w.D, code)), device)
        extra = w.B * w.T * 4 + w.D * 4                 # gaps and rates
        sgr.mingru_scan_decay(p, q, init, gaps, lam, out=out, workspace=wsd)
        if args.pass_ == "decay":
            fn = lambda: sgr.mingru_scan_decay(p, q, init, gaps, lam, out=out, workspace=wsd)  # noqa: E731
            bytes_step = w.algorithmic_bytes() + extra
            kernel_name = profile_kernel(sgr._abi.plan(0, w.B, w.T, w.D, code, True, decay=True))
        else:
            gy = torch.randn(p.shape, device=device, generator=g).to(p.dtype)
            fn = lambda: sgr.mingru_scan_decay_backward(p, q, init, gaps, lam, out, gy,  # noqa: E731
                                                        workspace=wsd)
            bytes_step = 6 * w.n_elems * w.elem_bytes + extra + w.D * 4 + \
                (2 * w.B * w.D * w.elem_bytes if init is not None else 0)
            kernel_name = backward_kernel(w)
        profile_key = w.name.replace("mingru_", "mingru_decay_", 1)
        ws = wsd
        args.no_e2e = True

    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    clocks = ClockSampler(local).start()
    barrier(world, device)
    torch.cuda.synchronize()
    h0 = time.time()
    total, per_launch = timed_launches(fn, args.steps, stream, while_busy=clocks.sample_now)
    h1 = time.time()
    barrier(world, device)
    clocks.stop()
    if ws.status() != 0:
        raise SystemExit("bench.py: a chunk timed out waiting for its carry (workspace status)")
    t_max = reduce_max(total, world, device)
    launch_max = reduce_max(per_launch, world, device)
    agg = aggregate(bytes_step, w.n_elems, args.steps, t_max, world)

    # end to end through the public API: pinned host inputs and output, the
    # library's time-sliced host scan (uploads, scans and downloads overlap)
    e2e = None
    if not args.no_e2e:
        hp = p.cpu().pin_memory()
        hq = q.cpu().pin_memory()
        hi = init.cpu().pin_memory() if init is not None else None
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        host_fn = sgr.mingru_scan_host if w.op == "mingru" else sgr.minmax_scan_host

        def e2e_step():
            host_fn(hp, hq, hi, out=hout, blocking=False)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world, device)
        e_steps = max(1, min(args.steps, 10))
        et, _ = timed_launches(e2e_step, e_steps, stream, lead=False)
        barrier(world, device)
        et = reduce_max(et, world, device)
        h2d = hp.numel() * hp.element_size() + hq.numel() * hq.element_size() + \
            (hi.numel() * hi.element_size() if hi is not None else 0)
        d2h = hout.numel() * hout.element_size()
        nbytes = sgr.staging_size(w.op, w.B, w.T, w.D, p.dtype)
        e2e = {"value": round(world * bytes_step * e_steps / et / 1e9, 2), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(et * 1e3 / e_steps, 3), "steps": e_steps,
               "api": f"{host_fn.__name__} (pinned host tensors in and out, time slices of "
                      "about sqrt(input MiB / 4.6) slices, uploads/scans/downloads overlapped)",
               "staging_bytes": nbytes}
        del hp, hq, hi, hout

    peak, peak_src = hbm_peak()
    achieved = bytes_step / launch_max / 1e9
    plan = sgr._abi.plan(0 if w.op == "mingru" else 1, w.B, w.T, w.D, 0 if w.dtype == "f32" else 1, True)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": UNIT,
                "frac": round(achieved / peak, 4), "traffic": recorded_traffic(profile_key, kernel_name.split("::")[1]),
                "peak_source": peak_src, "kernel": kernel_name,
                "bytes_per_launch": bytes_step,
                "launch_us": round(launch_max * 1e6, 2)}
    if args.pass_ == "projected":
        P = PROJECTED
        flops = 2.0 * P["B"] * P["T"] * P["d_in"] * 2 * P["D"]
        tpeak, tsrc = bf16_peak()
        roofline = {"bound": "tensor", "achieved": round(flops / launch_max / 1e12, 1), "peak": tpeak,
                    "unit": "TFLOP/s", "frac": round(flops / launch_max / 1e12 / tpeak, 4),
                    "traffic": recorded_traffic("b8_t4096_d1024_din1024", "mingru_projected_scan_kernel"),
                    "peak_source": tsrc, "kernel": kernel_name, "flops_per_launch": flops,
                    "launch_us": round(launch_max * 1e6, 2)}
    line = {
        "metric": METRIC, "value": round(agg["gbs"], 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(agg["ms_per_step"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic (seeded torch generator on the device)",
        "config": {"workload": w.name, "op": f"{w.op}_scan" + PASS_SUFFIX.get(args.pass_, ""),
                   "B": w.B, "T": w.T, "D": w.D,
                   "io_dtype": w.dtype, "initial_state": init is not None,
                   "global_batch": w.B * world, "seq_len": w.T, "parallelism": f"dp{world}",
                   "tile": f"{plan['tile_rows']}x{plan['tile_channels']}", "n_tiles": plan["n_tiles"],
                   "l2": "inputs larger than L2 (inputs + output per step "
                         f"{bytes_step / 1e6:.0f} MB vs 126 MB L2); no flush"},
        "gelem_per_s": round(agg["gelems"], 2),
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clocks.summary(h0, h1),
    }
    if args.pass_ == "projected":
        P = PROJECTED
        line["config"] = {"workload": "mingru_projected_b8_t4096_d1024_din1024", "op": "mingru_projected_scan",
                          "B": P["B"], "T": P["T"], "D": P["D"], "d_in": P["d_in"],
                          "io_dtype": "bf16 x and W in, f32 h out", "initial_state": True,
                          "global_batch": P["B"] * world, "seq_len": P["T"], "parallelism": f"dp{world}",
                          "tile": f"{PROJ_TILE[1]}x{PROJ_TILE[0]} (channels x tokens)",
                          "l2": "operands re-read per tile from L2; output larger than L2; no flush"}
        line["dtype"] = "bf16 products, f32 accumulation and scan"
        line["gelem_per_s"] = round(P["B"] * P["T"] * P["D"] * args.steps * world / total / 1e9, 2)
        line.pop("cpu_baseline", None)
        args.no_cpu = True
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(w, p, q, init)
    del p, q, init, out, ws
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_rows:
        rows = {}
        for name in WORKLOADS:
            if name != w.name:
                rows[name] = measure_row(WORKLOADS[name], device)
                torch.cuda.empty_cache()
        rows["mingru_step_b8_d1024_f32"] = measure_step_row(device)
        for name in ("mingru_b8_t4096_d1024_f32_h0", "minmax_b4_t8192_d768_f32",
                     "mingru_b16_t2048_d4096_bf16_h0"):
            rows[name.replace("_b", "_backward_b", 1)] = measure_backward_row(WORKLOADS[name], device)
            torch.cuda.empty_cache()
        for name in ("mingru_b8_t4096_d1024_f32_h0", "mingru_b16_t2048_d4096_bf16_h0"):
            rows.update(measure_decay_rows(WORKLOADS[name], device))
            torch.cuda.empty_cache()
        for name in ("mingru_b8_t4096_d1024_f32_h0", "mingru_b1_t131072_d512_f32_h0"):
            rows[name.replace("mingru_", "mingru_summary_", 1)] = measure_summary_row(WORKLOADS[name], device)
            torch.cuda.empty_cache()
        for name in ("mingru_b8_t4096_d1024_f32_h0", "mingru_b16_t2048_d4096_bf16_h0"):
            rows[name.replace("mingru_", "mingru_log_", 1)] = measure_log_row(WORKLOADS[name], device)
            torch.cuda.empty_cache()
        rows["mingru_projected_b8_t4096_d1024_din1024"] = measure_projected_row(device)
        torch.cuda.empty_cache()
        line["rows"] = rows
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args):
    """The CPU oracle timed as the reference arm, on bounded samples."""
    import oracle
    rank, world, local = dist_env()
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    if dev.type == "cuda":
        p, q, init = generate(w, device=dev)
    else:
        p, q, init = generate(w.scaled(B=1))
    cores = usable_cores()
    # one step = the oracle over one batch row (T x D elements) per thread
    rows = max(1, min(w.B, cores))
    ps, qs = p[:rows].cpu(), q[:rows].cpu()
    ins = init[:rows].cpu() if init is not None else None
    del p, q, init
    fn = oracle.mingru_linear if w.op == "mingru" else oracle.minmax
    for _ in range(args.warmup):
        fn(ps[:1, : max(1, w.T // 64)], qs[:1, : max(1, w.T // 64)],
           ins[:1] if ins is not None else None)
    times = []
    for _ in range(args.steps):
        t = time.perf_counter()
        fn(ps, qs, ins, threads=rows)
        times.append(time.perf_counter() - t)
    wall = sum(times)
    bytes_step = 3 * rows * w.T * w.D * w.elem_bytes + (rows * w.D * w.elem_bytes if ins is not None else 0)
    value = bytes_step * args.steps / wall / 1e9
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(wall / args.steps * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded torch generator)", "impl": "reference",
        "config": {"workload": w.name, "op": f"{w.op}_scan" + PASS_SUFFIX.get(args.pass_, ""),
                   "B": w.B, "T": w.T, "D": w.D,
                   "io_dtype": w.dtype, "initial_state": ins is not None, "global_batch": w.B,
                   "seq_len": w.T, "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": rows, "kind": "oracle",
                         "sample": f"each step: batch rows 0..{rows - 1} ({rows}x{w.T}x{w.D} elements) "
                                   f"of the workload, fp64 oracle, {rows} thread(s)"},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=BENCH_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--pass", dest="pass_", default="forward",
                    choices=["forward", "backward", "decay", "decay_backward", "projected", "log"],
                    help="time the scan (default), its gradient kernel on the workload, the time-decayed "
                         "minGRU or its gradient on the workload, the input projection fused with the "
                         "scan (B8 T4096 D1024 d_in 1024), or the minGRU scan evaluated in log space")
    ap.add_argument("--no-rows", action="store_true", help="skip the other hot-path rows")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    _, world, _ = dist_env()
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_b200(args)


if __name__ == "__main__":
    main()
