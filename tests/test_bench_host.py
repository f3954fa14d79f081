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


def test_decay_kernel_names():
    # the decayed scan keeps the plain plan's kernel except the channel-sequential one
    assert bench.decay_kernel({"kernel": 4}) == "sgr::scan_pipelined_kernel"
    assert bench.decay_kernel({"kernel": 3}) == "sgr::scan_pipelined_kernel"
    assert bench.decay_kernel({"kernel": 1}) == "sgr::scan_tile_kernel"


def test_cpu_baseline_record():
    w = Workload("t", "mingru", 2, 64, 32, "f32", seed=3, init="u01_1")
    p, q, i0 = generate(w)
    r = bench.cpu_baseline(w, p, q, i0, budget_s=0.5, cpu_target_s=0.05)
    assert r["kind"] == "oracle" and r["unit"] == bench.UNIT
    assert r["value"] > 0 and r["cores"] >= 1 and 1 <= r["passes"] <= 50
    assert r["cpu_seconds"] >= 0 and "batch rows" in r["sample"]
