"""GPU parity of the channel-sequential gradient kernel against the fp64
gradient oracle.

For wide batches each warp walks its 32 channels from t = T - 1 down to 0,
carrying dL/d(state) in a register.  Forced here (kernel override 4) on small
ragged shapes -- a partial top slot, T = 1, D not a multiple of the channel
group -- for the minGRU and MinMax gradients and the time-decayed minGRU's
(dL/dlambda included), with and without an initial state; a wide shape checks
the automatic choice.  Bars as for the other gradient kernels: error relative
to each channel's largest gradient, <= 1e-5 fp32 I/O, <= 2e-2 bf16 I/O; the
kernels read the oracle's forward output rounded to the I/O dtype.
"""
import numpy as np
import pytest
import torch

import oracle
import scan_gated_rnns_b200 as sgr
from scan_gated_rnns_b200 import _abi
from scan_gated_rnns_b200.synth import Workload, generate

from parity import TORCH_DT

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = torch.device("cuda:0")
TOL_BWD = {"f32": 1e-5, "bf16": 2e-2}
SEQ = _abi.KERNEL_SEQUENTIAL


@pytest.fixture(autouse=True)
def _reset_hooks():
    yield
    _abi.lib().sgr_set_kernel_override(0)


def channel_scaled_err(got, ref) -> float:
    """max over elements of |got - ref| / (largest |ref| of the element's
    channel).  With fewer than 8 steps a channel has too few elements to set a
    scale (minGRU's dk carries the factor g(hx) - h, which can cancel in a
    single element), so there the scale is the largest |ref| of the batch row."""
    got = got.detach().to("cpu", torch.float64).numpy()
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape
    if not np.isfinite(got).all():
        return float("inf")
    if ref.ndim == 3:
        axes = (1,) if ref.shape[1] >= 8 else (1, 2)
        scale = np.abs(ref).max(axis=axes, keepdims=True)
    else:
        scale = np.abs(ref)
    return float((np.abs(got - ref) / np.maximum(scale, 1e-30)).max())


def inputs(op, B, T, D, dtype, init, seed):
    p, q, i0 = generate(Workload("t", op, B, T, D, dtype, seed=seed, init=init))
    gy = torch.randn(B, T, D, generator=torch.Generator().manual_seed(seed + 1000)).to(TORCH_DT[dtype])
    fwd = oracle.mingru_linear(p, q, i0) if op == "mingru" else oracle.minmax(p, q, i0)
    return p, q, i0, torch.from_numpy(fwd).to(TORCH_DT[dtype]), gy


def dev(*ts):
    return [None if t is None else t.to(DEV) for t in ts]


SHAPES = [(2, 1, 64), (3, 17, 40), (2, 300, 96), (1, 1000, 200), (2, 2049, 136)]


@pytest.mark.parametrize("op", ["mingru", "minmax"])
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("init", [None, "u01_1"])
def test_sequential_backward_matches_oracle(op, shape, dtype, init):
    sgr.set_kernel_override(SEQ)
    p, q, i0, fwd, gy = inputs(op, *shape, dtype, init, seed=sum(shape) % 977)
    fn = sgr.mingru_scan_backward if op == "mingru" else sgr.minmax_scan_backward
    dp, dq, dinit = fn(*dev(p, q, i0, fwd, gy))
    torch.cuda.synchronize()
    ofn = oracle.mingru_backward if op == "mingru" else oracle.minmax_backward
    rp, rq, rinit = ofn(p, q, i0, gy, threads=8)
    assert dp.dtype == TORCH_DT[dtype] and dp.shape == p.shape
    assert channel_scaled_err(dp, rp) <= TOL_BWD[dtype]
    assert channel_scaled_err(dq, rq) <= TOL_BWD[dtype]
    # the initial-state gradient (a signed sum over the sequence), against the
    # largest |dL/dh0| of its batch row
    got = dinit.double().cpu().numpy()
    scale = np.maximum(np.abs(rinit).max(axis=1, keepdims=True), 1e-30)
    assert float((np.abs(got - rinit) / scale).max()) <= TOL_BWD[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("log1p_delta", [False, True])
def test_sequential_decay_backward_matches_oracle(dtype, log1p_delta):
    sgr.set_kernel_override(SEQ)
    B, T, D = 3, 500, 136
    k, hx, h0 = generate(Workload("t", "mingru", B, T, D, dtype, seed=91, init="u01_1"))
    g = torch.Generator().manual_seed(92)
    dt = torch.empty(B, T).exponential_(1.0 / (20.0 if log1p_delta else 0.5), generator=g)
    dt[:, T // 3] = 3e4                                   # wipes the state
    lam = torch.rand(D, generator=g) * 2.0
    gy = torch.randn(B, T, D, generator=g).to(TORCH_DT[dtype])
    fwd = torch.from_numpy(oracle.mingru_decay(k, hx, h0, dt, lam, log1p_delta)).to(TORCH_DT[dtype])
    dk, dhx, dh0, dlam = sgr.mingru_scan_decay_backward(*dev(k, hx, h0, dt, lam, fwd, gy), log1p_delta)
    torch.cuda.synchronize()
    rk, rhx, rh0, rlam = oracle.mingru_decay_backward(k, hx, h0, dt, lam, gy, log1p_delta)
    assert channel_scaled_err(dk, rk) <= TOL_BWD[dtype]
    assert channel_scaled_err(dhx, rhx) <= TOL_BWD[dtype]
    _, _, _, mag = oracle.mingru_decay_backward(k, hx, h0, dt, lam, np.abs(gy.double().numpy()), log1p_delta)
    scale = np.maximum(np.abs(mag), 1e-30)
    assert float((np.abs(dlam.cpu().double().numpy() - rlam) / scale).max()) <= TOL_BWD[dtype]


def test_wide_batch_gradient_selects_it_and_matches():
    B, T, D = 16, 48, 4096                                # 2048 channel groups: sequential
    pl_groups = B * (D // 32)
    assert pl_groups >= 9 * 148
    p, q, i0, fwd, gy = inputs("mingru", B, T, D, "bf16", "u01_1", seed=93)
    dp, dq, dinit = sgr.mingru_scan_backward(*dev(p, q, i0, fwd, gy))
    torch.cuda.synchronize()
    rp, rq, rinit = oracle.mingru_backward(p, q, i0, gy, threads=8)
    assert channel_scaled_err(dp, rp) <= TOL_BWD["bf16"]
    assert channel_scaled_err(dq, rq) <= TOL_BWD["bf16"]
    # the same gradient through the chunked tile kernel agrees
    sgr.set_kernel_override(_abi.KERNEL_TILE)
    tp, tq, tinit = sgr.mingru_scan_backward(*dev(p, q, i0, fwd, gy))
    torch.cuda.synchronize()
    assert channel_scaled_err(tp, rp) <= TOL_BWD["bf16"]
    # both initial-state gradients against the oracle's, per batch row
    for d0 in (dinit, tinit):
        got = d0.double().cpu().numpy()
        assert float((np.abs(got - rinit) / np.abs(rinit).max(axis=1, keepdims=True)).max()) <= TOL_BWD["bf16"]
