"""Build the CUDA library ``libsgr.so`` in-tree with nvcc for sm_100a.

    python -m scan_gated_rnns_b200.build [--force] [--verbose]

The library is rebuilt when any source under ``csrc/`` or the public header
is newer than it.  ``--verbose`` adds ``-Xptxas -v`` (registers, spills and
shared memory per kernel).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsgr.so")
STEP_EXE = os.path.join(PKG, "step_latency")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
         "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-Xcompiler", "-Wall"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libsgr.so")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in _deps())


def build(force: bool = False, verbose: bool = False) -> str:
    if force or verbose or not up_to_date():
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [nvcc(), *ARCH, *FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", tmp, *sources()]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    build_step_latency(force)
    return LIB


def build_step_latency(force: bool = False) -> str:
    """The host-loop decode timer (native/step_latency.cpp), a plain C++
    program linked against libsgr.so (found next to it at run time)."""
    src = os.path.join(PKG, "native", "step_latency.cpp")
    if not force and os.path.exists(STEP_EXE) and \
            os.path.getmtime(STEP_EXE) >= max(os.path.getmtime(src), os.path.getmtime(LIB)):
        return STEP_EXE
    tmp = STEP_EXE + f".tmp{os.getpid()}"
    cmd = [nvcc(), "-O2", "-std=c++17", "-x", "cu", "-gencode", "arch=compute_100a,code=sm_100a",
           "-I", INCLUDE, "-o", tmp, src, "-L", PKG, "-lsgr", "-Xlinker", "-rpath=$ORIGIN"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, STEP_EXE)
    return STEP_EXE


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
