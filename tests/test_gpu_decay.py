"""GPU parity of the time-decay minGRU (mingru_scan_decay, its gradient and
the autograd wrapper) against the fp64 decay oracle.

Decay contract (page "Your first delta model", Step 5, read for a vector
state): h_t = (1 - z_t) gamma_t h_{t-1} + z_t g(hx_t), gamma = exp(-lambda u),
u = delta_t or log1p(delta_t), lambda u > 1e4 wipes the state.  Forward bar:
max relative error <= 1e-5 fp32 I/O, <= 2e-2 bf16 I/O (the gaps and rates
are fp32 either way).  Gradients: error relative to each channel's largest
gradient, as for the plain gradients; dL/dlambda (sums over the batch and
time, accumulated with atomic adds) relative to the sum of the magnitudes of
its terms.
"""
import numpy as np
import pytest
import torch

import oracle
import scan_gated_rnns_b200 as sgr
from scan_gated_rnns_b200 import _abi
from scan_gated_rnns_b200.synth import Workload, generate

from parity import TOL, TORCH_DT, rel_err

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = torch.device("cuda:0")
TOL_BWD = {"f32": 1e-5, "bf16": 2e-2}


@pytest.fixture(autouse=True)
def _reset_hooks():
    yield
    lib = _abi.lib()
    lib.sgr_set_tile_override(0, 0)
    lib.sgr_set_kernel_override(0)


def channel_scaled_err(got, ref) -> float:
    got = got.detach().to("cpu", torch.float64).numpy() if hasattr(got, "detach") else np.asarray(got)
    scale = np.abs(ref).max(axis=1, keepdims=True)
    if not np.isfinite(got).all():
        return float("inf")
    return float((np.abs(got - ref) / np.maximum(scale, 1e-30)).max())


def data(B, T, D, dtype, init, seed, gap_scale=1.0, wipe_at=None):
    k, hx, h0 = generate(Workload("t", "mingru", B, T, D, dtype, seed=seed, init=init))
    g = torch.Generator().manual_seed(seed + 500)
    dt = torch.empty(B, T).exponential_(1.0 / gap_scale, generator=g)
    if wipe_at is not None:
        dt[:, wipe_at] = 3e4
    lam = torch.rand(D, generator=g) * 2.0
    return k, hx, h0, dt, lam


SHAPES = [(2, 1024, 512), (3, 1000, 96), (1, 777, 36), (2, 300, 7), (1, 1, 1), (1, 4097, 32)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("init", [None, "u01_1"])
@pytest.mark.parametrize("log1p_delta", [False, True])
def test_decay_forward_matches_oracle(shape, dtype, init, log1p_delta):
    k, hx, h0, dt, lam = data(*shape, dtype, init, seed=sum(shape) % 101,
                              gap_scale=20.0 if log1p_delta else 0.5,
                              wipe_at=shape[1] // 2 if shape[1] > 2 else None)
    h = sgr.mingru_scan_decay(k.to(DEV), hx.to(DEV), None if h0 is None else h0.to(DEV),
                              dt.to(DEV), lam.to(DEV), log1p_delta)
    torch.cuda.synchronize()
    ref = oracle.mingru_decay(k, hx, h0, dt, lam, log1p_delta)
    assert h.dtype == TORCH_DT[dtype]
    assert rel_err(h, ref) <= TOL[dtype]


# (kernel, rows per thread): tile kernel, 7- and 15-warp pipelined kernels
# (8 rows per thread: bf16 only, the automatic choice there)
@pytest.mark.parametrize("kernel,r", [(1, 2), (1, 4), (2, 2), (2, 4), (3, 4), (2, 8), (3, 8)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decay_every_kernel(kernel, r, dtype):
    if r == 8 and dtype == "f32":
        pytest.skip("fp32 tiles take at most 4 rows per thread")
    sgr.set_kernel_override(kernel)
    sgr.set_tile_override(0, r)
    k, hx, h0, dt, lam = data(3, 2500, 160, dtype, "u01_1", seed=kernel * 7 + r, wipe_at=1300)
    h = sgr.mingru_scan_decay(k.to(DEV), hx.to(DEV), h0.to(DEV), dt.to(DEV), lam.to(DEV))
    torch.cuda.synchronize()
    assert rel_err(h, oracle.mingru_decay(k, hx, h0, dt, lam)) <= TOL[dtype]


# Wide batches: the decayed scan takes the channel-sequential kernel the
# plain scan's plan names (gaps spread across the lanes one slot ahead), its
# workspace is the status header, and no wait gives up.
@pytest.mark.parametrize("dtype,B", [("f32", 16), ("bf16", 24), ("bf16", 64)])
@pytest.mark.parametrize("log1p_delta", [False, True])
def test_decay_wide_batch(dtype, B, log1p_delta):
    T, D = 300, 2048
    code = _abi.SGR_F32 if dtype == "f32" else _abi.SGR_BF16
    pl = _abi.plan(_abi.SGR_OP_MINGRU, B, T, D, code, True, decay=True)
    plain = _abi.plan(_abi.SGR_OP_MINGRU, B, T, D, code, True)["kernel"]
    # bf16 from 16 groups per SM: four warps per 64-channel group
    assert pl["kernel"] == (_abi.KERNEL_SEQUENTIAL_QUAD if dtype == "bf16" and B * D / 32 >= 16 * 148 else plain)
    assert pl["kernel"] in (_abi.KERNEL_SEQUENTIAL, _abi.KERNEL_SEQUENTIAL_PAIR, _abi.KERNEL_SEQUENTIAL_QUAD)
    need = sgr.workspace_size("mingru", B, T, D, TORCH_DT[dtype])
    assert need >= pl["workspace_bytes"]
    k, hx, h0, dt, lam = data(B, T, D, dtype, "u01_1", seed=B, wipe_at=150,
                              gap_scale=20.0 if log1p_delta else 1.0)
    ws = sgr.Workspace(need, DEV)
    h = sgr.mingru_scan_decay(k.to(DEV), hx.to(DEV), h0.to(DEV), dt.to(DEV), lam.to(DEV), log1p_delta,
                              workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == _abi.SGR_OK
    assert rel_err(h, oracle.mingru_decay(k, hx, h0, dt, lam, log1p_delta)) <= TOL[dtype]


# Gaps and rates through the copy engine (16-byte aligned starts, a batch
# stride that is a multiple of 4) or, otherwise, plain loads: a padded
# stride, an odd one, an unaligned start of the gaps or of the rates, and a
# single batch row whose length is not a multiple of 4.
@pytest.mark.parametrize("B,pad,gap_off,lam_off", [(3, 3, 0, 0), (3, 1, 0, 0), (3, 0, 1, 0),
                                                   (3, 3, 0, 1), (1, 0, 0, 0)])
@pytest.mark.parametrize("kernel", [0, 2, 3])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decay_gap_layouts(B, pad, gap_off, lam_off, kernel, dtype):
    if kernel == 0 and dtype == "bf16":
        pytest.skip("the automatic bf16 plans take the tile kernels at this size")
    sgr.set_kernel_override(kernel)
    sgr.set_tile_override(0, 4)
    # the automatic fp32 plan takes two 6-warp blocks per SM from two tiles
    # per block (592 tiles of 96 rows): 3 x 20 chains of 32 channels
    T, D = 2501, 640 if kernel == 0 else 160
    k, hx, h0, dt, lam = data(B, T, D, dtype, "u01_1", seed=11 + pad + gap_off + lam_off, wipe_at=1200)
    gstore = torch.full((B, T + pad + gap_off), float("nan"), device=DEV)
    gaps = gstore[:, gap_off:gap_off + T]
    gaps.copy_(dt.to(DEV))
    lstore = torch.full((D + lam_off,), float("nan"), device=DEV)
    rates = lstore[lam_off:]
    rates.copy_(lam.to(DEV))
    h = sgr.mingru_scan_decay(k.to(DEV), hx.to(DEV), h0.to(DEV), gaps, rates)
    torch.cuda.synchronize()
    assert rel_err(h, oracle.mingru_decay(k, hx, h0, dt, lam)) <= TOL[dtype]
    # the pipelined gradient (2: 7-warp blocks, 3: 15-warp blocks; 0: the
    # automatic plan, two 6-warp blocks per SM with three batch rows, one
    # 7-warp block per SM with one) with the same layouts: gaps and rates in
    # its ring slots or by plain loads
    assert _abi.lib().sgr_backward_kernel(0, B, T, D, _abi.SGR_F32 if dtype == "f32" else _abi.SGR_BF16, 1) == 2
    g = torch.Generator().manual_seed(13 + pad)
    gy = torch.randn(B, T, D, generator=g).to(TORCH_DT[dtype])
    fwd = torch.from_numpy(oracle.mingru_decay(k, hx, h0, dt, lam)).to(TORCH_DT[dtype])
    dk, dhx, dh0, dlam = sgr.mingru_scan_decay_backward(k.to(DEV), hx.to(DEV), h0.to(DEV), gaps, rates,
                                                        fwd.to(DEV), gy.to(DEV))
    torch.cuda.synchronize()
    rk, rhx, rh0, rlam = oracle.mingru_decay_backward(k, hx, h0, dt, lam, gy)
    assert channel_scaled_err(dk, rk) <= TOL_BWD[dtype]
    assert channel_scaled_err(dhx, rhx) <= TOL_BWD[dtype]
    e0 = float((np.abs(dh0.cpu().double().numpy() - rh0) / np.abs(rh0).max(axis=1, keepdims=True)).max())
    assert e0 <= TOL_BWD[dtype]
    assert lam_err(dlam, rlam, k, hx, h0, dt, lam, gy) <= TOL_BWD[dtype]


@pytest.mark.parametrize("log1p_delta", [False, True])
def test_decay_workload_gradient_every_channel(log1p_delta):
    """The decayed gradient on the B8 x 4096 x 1024 fp32 workload (the
    pipelined gradient, two 6-warp blocks per SM, gaps and rates in its ring
    slots) against the oracle on every channel."""
    B, T, D = 8, 4096, 1024
    assert _abi.lib().sgr_backward_kernel(0, B, T, D, _abi.SGR_F32, 1) == 2
    k, hx, h0, dt, lam = data(B, T, D, "f32", "u01_1", seed=61, gap_scale=20.0 if log1p_delta else 1.0,
                              wipe_at=2000)
    g = torch.Generator().manual_seed(62)
    gy = torch.randn(B, T, D, generator=g)
    fwd = torch.from_numpy(oracle.mingru_decay(k, hx, h0, dt, lam, log1p_delta)).float()
    dk, dhx, dh0, dlam = sgr.mingru_scan_decay_backward(k.to(DEV), hx.to(DEV), h0.to(DEV), dt.to(DEV),
                                                        lam.to(DEV), fwd.to(DEV), gy.to(DEV), log1p_delta)
    torch.cuda.synchronize()
    rk, rhx, rh0, rlam = oracle.mingru_decay_backward(k, hx, h0, dt, lam, gy, log1p_delta)
    ek, eh = channel_scaled_err(dk, rk), channel_scaled_err(dhx, rhx)
    e0 = float((np.abs(dh0.cpu().double().numpy() - rh0) / np.abs(rh0).max(axis=1, keepdims=True)).max())
    gabs = np.abs(gy.double().numpy())
    _, _, _, mag = oracle.mingru_decay_backward(k, hx, h0, dt, lam, gabs, log1p_delta)
    el = float((np.abs(dlam.cpu().double().numpy() - rlam) / np.maximum(np.abs(mag), 1e-30)).max())
    print(f"decayed gradient B8 x 4096 x 1024 log1p={log1p_delta}: dk {ek:.3e}, dhx {eh:.3e}, "
          f"dh0 {e0:.3e} (scaled), dlam {el:.3e} of the summed term magnitudes")
    assert max(ek, eh, e0, el) <= TOL_BWD["f32"]


# The channel-sequential kernels take the gaps through the copy engine when
# the gap array allows it (16-byte aligned start, batch stride a multiple of
# 4) and load them themselves otherwise: both, forward and gradient.
@pytest.mark.parametrize("B,pad,gap_off", [(3, 0, 0), (3, 3, 0), (3, 1, 0), (3, 0, 1), (1, 0, 0)])
@pytest.mark.parametrize("kernel", [4, 5, 6, 7, 8])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decay_sequential_gap_layouts(B, pad, gap_off, kernel, dtype):
    sgr.set_kernel_override(kernel)
    T, D = 1001, 96
    k, hx, h0, dt, lam = data(B, T, D, dtype, "u01_1", seed=21 + pad + gap_off + kernel, wipe_at=500)
    gstore = torch.full((B, T + pad + gap_off), float("nan"), device=DEV)
    gaps = gstore[:, gap_off:gap_off + T]
    gaps.copy_(dt.to(DEV))
    h = sgr.mingru_scan_decay(k.to(DEV), hx.to(DEV), h0.to(DEV), gaps, lam.to(DEV))
    torch.cuda.synchronize()
    assert rel_err(h, oracle.mingru_decay(k, hx, h0, dt, lam)) <= TOL[dtype]
    # the gradient (channel-sequential for these kinds) with the same gap layout
    g = torch.Generator().manual_seed(9)
    gy = torch.randn(B, T, D, generator=g).to(TORCH_DT[dtype])
    fwd = torch.from_numpy(oracle.mingru_decay(k, hx, h0, dt, lam)).to(TORCH_DT[dtype])
    dk, dhx, dh0, dlam = sgr.mingru_scan_decay_backward(k.to(DEV), hx.to(DEV), h0.to(DEV), gaps, lam.to(DEV),
                                                        fwd.to(DEV), gy.to(DEV))
    torch.cuda.synchronize()
    rk, rhx, rh0, rlam = oracle.mingru_decay_backward(k, hx, h0, dt, lam, gy)
    assert channel_scaled_err(dk, rk) <= TOL_BWD[dtype]
    assert channel_scaled_err(dhx, rhx) <= TOL_BWD[dtype]
    assert lam_err(dlam, rlam, k, hx, h0, dt, lam, gy) <= TOL_BWD[dtype]


def test_decay_zero_gaps_equal_plain_scan():
    k, hx, h0, dt, lam = data(2, 3000, 256, "f32", "u01_1", seed=3)
    z = torch.zeros_like(dt)
    a = sgr.mingru_scan_decay(k.to(DEV), hx.to(DEV), h0.to(DEV), z.to(DEV), lam.to(DEV))
    b = sgr.mingru_scan(k.to(DEV), hx.to(DEV), h0.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(a, b)    # gamma = 2^0 = 1 exactly: the same arithmetic


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("init", [None, "u01_1"])
@pytest.mark.parametrize("shape", [(2, 1000, 96), (1, 3001, 40), (3, 200, 7)])
def test_decay_backward_matches_oracle(dtype, init, shape):
    k, hx, h0, dt, lam = data(*shape, dtype, init, seed=sum(shape) % 89, wipe_at=shape[1] // 3)
    g = torch.Generator().manual_seed(77)
    gy = torch.randn(*shape, generator=g).to(TORCH_DT[dtype])
    fwd = torch.from_numpy(oracle.mingru_decay(k, hx, h0, dt, lam)).to(TORCH_DT[dtype])
    dk, dhx, dh0, dlam = sgr.mingru_scan_decay_backward(
        *(None if t is None else t.to(DEV) for t in (k, hx, h0, dt, lam, fwd, gy)))
    torch.cuda.synchronize()
    rk, rhx, rh0, rlam = oracle.mingru_decay_backward(k, hx, h0, dt, lam, gy)
    assert channel_scaled_err(dk, rk) <= TOL_BWD[dtype]
    assert channel_scaled_err(dhx, rhx) <= TOL_BWD[dtype]
    # dlam_d sums B T signed terms: its error is measured against the sum of
    # the terms' magnitudes (the oracle's dlam for |gy|, every term >= 0)
    err = lam_err(dlam, rlam, k, hx, h0, dt, lam, gy)
    print(f"decay gradient {shape} {dtype} init={init}: dlam error {err:.3e} of the summed term magnitudes")
    assert err <= TOL_BWD[dtype]


def lam_err(got, rlam, k, hx, h0, dt, lam, gy) -> float:
    """max_d |got_d - ref_d| / sum over (b, t) of |term_bt,d|: the oracle's
    dL/dlambda for |gy| is that sum (every term then has the same sign)."""
    gabs = np.abs(gy.double().numpy() if hasattr(gy, "double") else np.asarray(gy, np.float64))
    _, _, _, mag = oracle.mingru_decay_backward(k, hx, h0, dt, lam, gabs)
    got = got.detach().cpu().double().numpy() if hasattr(got, "detach") else np.asarray(got, np.float64)
    return float((np.abs(got - rlam) / np.maximum(np.abs(mag), 1e-30)).max())


def test_decay_autograd_wrapper_learns_lambda():
    B, T, D = 2, 800, 64
    k, hx, h0, dt, lam = data(B, T, D, "f32", "u01_1", seed=41)
    gy = torch.randn(B, T, D, generator=torch.Generator().manual_seed(4))
    K, H, H0, L = (t.to(DEV).requires_grad_() for t in (k, hx, h0, lam))
    y = sgr.mingru_scan_decay_fn(K, H, H0, dt.to(DEV), L)
    (y * gy.to(DEV)).sum().backward()
    rk, rhx, rh0, rlam = oracle.mingru_decay_backward(k, hx, h0, dt, lam, gy)
    assert channel_scaled_err(K.grad, rk) <= TOL_BWD["f32"]
    assert channel_scaled_err(H.grad, rhx) <= TOL_BWD["f32"]
    # dL/dh0 (a signed sum over the sequence) against the largest |dL/dh0| of
    # its batch row; dL/dlambda against its summed term magnitudes
    g0 = H0.grad.cpu().double().numpy()
    e0 = float((np.abs(g0 - rh0) / np.abs(rh0).max(axis=1, keepdims=True)).max())
    el = lam_err(L.grad, rlam, k, hx, h0, dt, lam, gy)
    print(f"decay autograd: dh0 error {e0:.3e} (row-scaled), dlam error {el:.3e} (term-magnitude-scaled)")
    assert e0 <= TOL_BWD["f32"] and el <= TOL_BWD["f32"]
