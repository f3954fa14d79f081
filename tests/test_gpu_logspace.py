"""mingru_scan_log: the minGRU scan evaluated in log space (page "Mingru
Pytorch", Requirements & limits: the log-space numerically stable minGRU),
through the C ABI, against the oracle's term-by-term log-space formula and its
linear recurrence on every channel.

Covered: the tile kernel (unaligned rows, few tiles), the pipelined kernels
(forced 7- and 15-warp blocks, several row counts), an absent initial state
(log h = -inf until the first token), an initial state with zero rows, a
sequence of one chunk and the full-size fp32 and bf16 shapes of the linear
parity tests.  The bar is the linear kernels' (1e-5 fp32, 2e-2 bf16): each
step adds two MUFU log/exp approximations (about 2^-22 each) to log2 h, an
absolute error in the log that is a relative one in h, and the state forgets
it at the rate the gates close, so it stays near the fp32 rounding of the
linear pairs; the tests print the error reached.
"""
import numpy as np
import pytest
import torch

import oracle
import scan_gated_rnns_b200 as sgr
from scan_gated_rnns_b200 import _abi
from scan_gated_rnns_b200.synth import WORKLOADS, Workload, generate

from parity import TOL, full_rel_err, rel_err

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = torch.device("cuda:0")


@pytest.fixture(autouse=True)
def _reset_override():
    yield
    sgr.set_kernel_override(0)


def unaligned(x):
    buf = torch.empty(x.numel() + 1, dtype=x.dtype, device=x.device)
    v = buf[1:].view(x.shape)
    v.copy_(x)
    return v


def run_log(k, hx, h0, shift=False):
    kd, hd = k.to(DEV), hx.to(DEV)
    h0d = None if h0 is None else h0.to(DEV)
    if shift:
        kd, hd = unaligned(kd), unaligned(hd)
    out = torch.full(kd.shape, float("nan"), dtype=kd.dtype, device=DEV)
    if shift:
        out = unaligned(out)
    ws = sgr.Workspace(sgr.workspace_size("mingru_log", *kd.shape, kd.dtype), DEV)
    sgr.mingru_scan_log(kd, hd, h0d, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == _abi.SGR_OK
    return out


CASES = [
    # (B, T, D, dtype, h0, shift, override)
    (2, 1000, 96, "f32", "u01_1", True, 0),      # scalar tile kernel
    (3, 777, 64, "f32", None, False, 1),         # vector tile kernel, no initial state
    (4, 3000, 256, "f32", "u01_1", False, 2),    # pipelined, 7-warp blocks
    (4, 3000, 256, "f32", "u01_1", False, 3),    # pipelined, 15-warp blocks
    (4, 3000, 256, "bf16", "u01_1", False, 2),
    (2, 5000, 512, "bf16", None, False, 3),
    (5, 100, 128, "f32", "u01_1", False, 2),     # one chunk per chain
]


@pytest.mark.parametrize("B,T,D,dt,init,shift,kern", CASES)
def test_log_scan_matches_the_log_space_oracle(B, T, D, dt, init, shift, kern):
    sgr.set_kernel_override(kern)
    w = Workload("log", "mingru", B, T, D, dt, seed=B * 7 + T, init=init)
    k, hx, h0 = generate(w)
    got = run_log(k, hx, h0, shift)
    ref = oracle.mingru_log(k.double().numpy(), hx.double().numpy(),
                            None if h0 is None else h0.double().numpy(), threads=8)
    err = rel_err(got, ref)
    lin = oracle.mingru_linear(k.double().numpy(), hx.double().numpy(),
                               None if h0 is None else h0.double().numpy(), threads=8)
    print(f"log-space scan {B}x{T}x{D} {dt} kernel {kern}: max relative error {err:.3e}")
    assert err <= TOL[dt]
    assert rel_err(got, lin) <= TOL[dt]


def test_log_scan_initial_state_rows_of_zero():
    # h0 = 0 carries log h = -inf into the first step: the same as no state
    B, T, D = 3, 2000, 128
    w = Workload("log0", "mingru", B, T, D, "f32", seed=5, init="u01_1")
    k, hx, h0 = generate(w)
    h0[1] = 0.0
    sgr.set_kernel_override(2)
    got = run_log(k, hx, h0)
    ref = oracle.mingru_linear(k.double().numpy(), hx.double().numpy(), h0.double().numpy(), threads=8)
    err = rel_err(got, ref)
    print(f"log-space scan with zero initial rows: max relative error {err:.3e}")
    assert err <= TOL["f32"]


@pytest.mark.parametrize("name", ["mingru_b8_t4096_d1024_f32_h0", "mingru_b16_t2048_d4096_bf16_h0"])
def test_log_scan_full_size_every_channel(name):
    w = WORKLOADS[name]
    k, hx, h0 = generate(w)
    got = run_log(k, hx, h0)
    err = full_rel_err("mingru", k, hx, h0, got, fn=oracle.mingru_log)
    print(f"{name} log-space scan: max relative error over every channel {err:.3e}")
    assert err <= TOL[w.dtype]


def test_log_scan_plan_is_chunked_and_sized():
    # wide batches: the linear scan runs one warp per channel group over the
    # whole sequence; the log-space scan is cut into chunks and needs words
    B, T, D = 16, 2048, 4096
    lin = _abi.plan(_abi.SGR_OP_MINGRU, B, T, D, _abi.SGR_BF16)
    log = _abi.plan(_abi.SGR_OP_MINGRU_LOG, B, T, D, _abi.SGR_BF16)
    assert lin["kernel"] in (_abi.KERNEL_SEQUENTIAL, _abi.KERNEL_SEQUENTIAL_PAIR, _abi.KERNEL_SEQUENTIAL_PAIR2,
                             _abi.KERNEL_SEQUENTIAL_QUAD)
    assert log["kernel"] in (_abi.KERNEL_PIPELINED, _abi.KERNEL_PIPELINED_WIDE)
    assert sgr.workspace_size("mingru_log", B, T, D, torch.bfloat16) >= log["workspace_bytes"] > 256
    assert np.isfinite(log["n_tiles"])
