"""Host-side pieces of bench.py, on CPU: the committed ncu summaries carry
the fields the JSON line reads, the kernel each plan launches is named, and
the CPU-baseline leg returns a complete record on a small workload."""
import glob
import os
import re

import pytest

import bench
from scan_gated_rnns_b200.synth import Workload, generate

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def summary_fields(path):
    fields = {}
    with open(path) as f:
        for line in f:
            if line.startswith("- ") and ":" in line:
                k, v = line[2:].split(":", 1)
                v = v.strip()
                fields[k.strip()] = v[1:].split("`", 1)[0] if v.startswith("`") else v
    return fields


@pytest.mark.parametrize("path", sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))))
def test_profile_summaries_carry_traffic_and_source_hash(path):
    name = os.path.basename(path)[:-3]
    kernels = [k for k in bench.KERNEL_SOURCES if name.startswith(k + "_")]
    assert kernels, f"{name}: not named after a kernel bench.py reports"
    f = summary_fields(path)
    assert re.fullmatch(r"[0-9a-f]{16}", f.get("kernel_source_sha", "")), name
    assert int(f["dram_bytes_per_launch"]) > 0
    text = open(path).read()
    # the command that made it, with clocks left alone, on committed files only
    assert "ncu --set full --clock-control none" in text and "python bench.py" in text
    assert "_work" not in text


def test_plan_kernel_names():
    assert bench.plan_kernel({"kernel": 1}) == "sgr::scan_tile_kernel"
    assert bench.plan_kernel({"kernel": 2}) == bench.plan_kernel({"kernel": 3}) == "sgr::scan_pipelined_kernel"
    assert bench.plan_kernel({"kernel": 4}) == "sgr::scan_sequential_kernel"


def test_usable_cores_follow_the_affinity_mask(monkeypatch):
    monkeypatch.setattr(bench.os, "sched_getaffinity", lambda pid: {0, 2, 5})
    assert bench.usable_cores() == 3
    monkeypatch.setattr(bench.os, "sched_getaffinity", lambda pid: set(range(100)))
    assert bench.usable_cores() == 32


def test_cpu_baseline_record():
    w = Workload("t", "mingru", 2, 64, 32, "f32", seed=3, init="u01_1")
    p, q, i0 = generate(w)
    r = bench.cpu_baseline(w, p, q, i0, budget_s=0.5, cpu_target_s=0.05)
    assert r["kind"] == "oracle" and r["unit"] == bench.UNIT
    assert r["value"] > 0 and r["cores"] >= 1 and 1 <= r["passes"] <= 50
    assert r["cpu_seconds"] >= 0 and "batch rows" in r["sample"]
    one = r["single_thread"]
    assert one["value"] > 0 and one["unit"] == bench.UNIT and "1 thread" in one["sample"]


def test_clock_samples_taken_inside_the_timed_region():
    # a fake NVML reading: samples from the calling thread carry the reasons
    # bits, and the summary keeps those inside the window
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.samples, c.ok, c.max_mhz = [], True, 1965
    c._read = lambda: (1965, 0x4, 500.0)
    t0 = bench.time.time()
    for _ in range(3):
        c.sample_now()
    t1 = bench.time.time()
    c.samples.append((t1 + 10.0, 900, 0x40, 100.0))      # after the window: ignored
    r = c.summary(t0, t1)
    assert r["samples"] == 3 and r["window"] == "timed region"
    assert r["sm_mhz"] == 1965 and r["reasons"] == ["sw_power_cap"] and r["power_w_max"] == 500.0
    # NVML missing: no samples, clocks reported as unknown
    c.ok = False
    c.sample_now()
    assert c.summary(t0, t1)["sm_mhz"] is None


def test_timed_launches_samples_until_the_stream_is_done(monkeypatch):
    # fake CUDA events: the end event completes after a few queries
    class Ev:
        polls = 0

        def __init__(self, enable_timing=True):
            pass

        def record(self, stream):
            pass

        def query(self):
            Ev.polls += 1
            return Ev.polls > 4

        def elapsed_time(self, other):
            return 2.0

    monkeypatch.setattr(bench.torch.cuda, "Event", Ev)
    monkeypatch.setattr(bench.torch.cuda, "synchronize", lambda: None)
    spins = []
    monkeypatch.setattr(bench.torch.cuda, "_sleep", lambda cycles: spins.append(cycles))
    calls, seen = [], []
    total, per = bench.timed_launches(lambda: calls.append(1), 3, None, while_busy=lambda: seen.append(1))
    assert len(calls) == 3 and len(seen) == 4
    assert total == 2e-3 and per == 2e-3
    assert spins == [bench.LEAD_CYCLES]                      # one spin ahead of the start event
    Ev.polls = 0
    bench.timed_launches(lambda: None, 2, None, lead=False)  # no sampler: no queries; no spin
    assert Ev.polls == 0 and spins == [bench.LEAD_CYCLES]

