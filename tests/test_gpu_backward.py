"""GPU parity of the gradient kernels (mingru_scan_backward,
minmax_scan_backward and the autograd wrappers) against the fp64 gradient
oracle, element by element.

The gradients are sums of signed terms (delta_t = gy_t + carried part, and
minGRU's dk has the factor g(hx) - h), so an element's relative error is not
bounded where terms cancel; the bar is the error relative to the largest
gradient of the same channel (the scale the floating-point sums work at):
max |gpu - ref| / max_t |ref| <= 1e-5 with fp32 I/O, <= 2e-2 with bf16 I/O
(outputs rounded to bf16).  The kernels read the forward output h; the tests
give them the oracle's forward rounded to the I/O dtype, never a GPU result.
"""
import numpy as np
import pytest
import torch

import oracle
import scan_gated_rnns_b200 as sgr
from scan_gated_rnns_b200 import _abi
from scan_gated_rnns_b200.synth import WORKLOADS, Workload, generate

from parity import TORCH_DT

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
    lib.sgr_set_wait_limit(0)
    lib.sgr_set_drop_publish(-1)


def channel_scaled_err(got, ref) -> float:
    """max over elements of |got - ref| / (largest |ref| of the element's channel)."""
    if hasattr(got, "detach"):
        got = got.detach().to("cpu", torch.float64).numpy()
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert got.shape == ref.shape
    if got.size == 0:
        return 0.0
    if not np.isfinite(got).all():
        return float("inf")
    if ref.ndim == 3:
        scale = np.abs(ref).max(axis=1, keepdims=True)
    else:
        scale = np.abs(ref)
    return float((np.abs(got - ref) / np.maximum(scale, 1e-30)).max())


def inputs(op, B, T, D, dtype, init, seed):
    w = Workload("t", op, B, T, D, dtype, seed=seed, init=init)
    p, q, i0 = generate(w)
    g = torch.Generator().manual_seed(seed + 1000)
    gy = torch.randn(B, T, D, generator=g).to(TORCH_DT[dtype])
    fwd = oracle.mingru_linear(p, q, i0) if op == "mingru" else oracle.minmax(p, q, i0)
    fwd = torch.from_numpy(fwd).to(TORCH_DT[dtype])
    return p, q, i0, fwd, gy


def gpu_backward(op, p, q, i0, fwd, gy, **kw):
    fn = sgr.mingru_scan_backward if op == "mingru" else sgr.minmax_scan_backward
    dev = [None if t is None else t.to(DEV) for t in (p, q, i0, fwd, gy)]
    out = fn(*dev, **kw)
    torch.cuda.synchronize()
    return out


def oracle_backward(op, p, q, i0, gy):
    fn = oracle.mingru_backward if op == "mingru" else oracle.minmax_backward
    return fn(p, q, i0, gy, threads=8)


SHAPES = [(2, 1024, 512), (3, 1000, 96), (1, 777, 36), (2, 300, 7), (1, 1, 1), (5, 1, 64),
          (1, 4097, 32), (2, 129, 40), (4, 63, 8), (1, 2000, 1)]


@pytest.mark.parametrize("op", ["mingru", "minmax"])
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("init", [None, "u01_1"])
def test_backward_matches_oracle(op, shape, dtype, init):
    p, q, i0, fwd, gy = inputs(op, *shape, dtype, init, seed=sum(shape) % 977)
    dp, dq, dinit = gpu_backward(op, p, q, i0, fwd, gy)
    rp, rq, rinit = oracle_backward(op, p, q, i0, gy)
    assert dp.dtype == TORCH_DT[dtype] and dp.shape == p.shape
    assert channel_scaled_err(dp, rp) <= TOL_BWD[dtype]
    assert channel_scaled_err(dq, rq) <= TOL_BWD[dtype]
    assert row_scaled_err(dinit, rinit) <= TOL_BWD[dtype]


def row_scaled_err(got, ref) -> float:
    """dL/d(initial state), (B, D): a signed sum over the whole sequence, so
    measured against the largest |dL/dh0| of the same batch row."""
    got = got.detach().double().cpu().numpy() if hasattr(got, "detach") else np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.maximum(np.abs(ref).max(axis=1, keepdims=True), 1e-30)
    return float((np.abs(got - ref) / scale).max())


# The pipelined gradient (persistent blocks, copy-engine ring; the automatic
# choice for aligned narrow batches with at least two tiles per SM), forced on
# shapes with ragged sequences and channel tiles, one-tile sequences, a single
# row and short sequences.
PIPE_SHAPES = [(2, 1000, 96), (1, 3001, 40), (3, 250, 160), (1, 121, 64), (2, 7, 32), (4, 240, 8)]


@pytest.mark.parametrize("op", ["mingru", "minmax"])
@pytest.mark.parametrize("shape", PIPE_SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("init", [None, "u01_1"])
@pytest.mark.parametrize("kernel", [2, 3])
def test_pipelined_backward_matches_oracle(op, shape, dtype, init, kernel):
    """kernel 2: blocks of 7 data warps (two per SM); 3: of 15 (one per SM)."""
    B, T, D = shape
    if dtype == "bf16" and D % 8:
        pytest.skip("bf16 vector rows need D % 8 == 0")
    sgr.set_kernel_override(kernel)
    code = _abi.SGR_F32 if dtype == "f32" else _abi.SGR_BF16
    assert _abi.lib().sgr_backward_kernel(0 if op == "mingru" else 1, B, T, D, code, 1) == 2
    p, q, i0, fwd, gy = inputs(op, *shape, dtype, init, seed=sum(shape) % 811 + 5)
    dp, dq, dinit = gpu_backward(op, p, q, i0, fwd, gy)
    rp, rq, rinit = oracle_backward(op, p, q, i0, gy)
    assert channel_scaled_err(dp, rp) <= TOL_BWD[dtype]
    assert channel_scaled_err(dq, rq) <= TOL_BWD[dtype]
    assert row_scaled_err(dinit, rinit) <= TOL_BWD[dtype]


@pytest.mark.parametrize("op", ["mingru", "minmax"])
@pytest.mark.parametrize("r", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_every_tile_shape(op, r, dtype):
    sgr.set_tile_override(0, r)
    p, q, i0, fwd, gy = inputs(op, 3, 1500, 160, dtype, "u01_1", seed=r)
    dp, dq, _ = gpu_backward(op, p, q, i0, fwd, gy)
    rp, rq, _ = oracle_backward(op, p, q, i0, gy)
    assert channel_scaled_err(dp, rp) <= TOL_BWD[dtype]
    assert channel_scaled_err(dq, rq) <= TOL_BWD[dtype]


def test_minmax_backward_ties_match_oracle():
    g = torch.Generator().manual_seed(3)
    vals = torch.tensor([-1.0, 0.0, 1.0, 2.0])
    B, T, D = 2, 3000, 40
    r = vals[torch.randint(0, 4, (B, T, D), generator=g)]
    s = vals[torch.randint(0, 4, (B, T, D), generator=g)]
    x0 = vals[torch.randint(0, 4, (B, D), generator=g)]
    gy = torch.randint(-8, 9, (B, T, D), generator=g).float()
    fwd = torch.from_numpy(oracle.minmax(r, s, x0)).float()
    dr, ds, dx0 = gpu_backward("minmax", r, s, x0, fwd, gy)
    rr, rs, rx0 = oracle.minmax_backward(r, s, x0, gy, threads=8)
    # ties everywhere: the coefficients 0, 1/4, 1/2, 1 are exact; only the sums round
    assert channel_scaled_err(dr, rr) <= TOL_BWD["f32"]
    assert channel_scaled_err(ds, rs) <= TOL_BWD["f32"]
    assert np.allclose(dx0.cpu().double().numpy(), rx0, rtol=1e-5, atol=1e-5)
    # where a step's operands are all distinct, the split is 0 or 1: gradient to one operand
    distinct = (r != s).numpy() & (r != torch.cat([x0[:, None], fwd[:, :-1]], 1)).numpy()
    both = (dr.cpu().numpy() != 0) & (ds.cpu().numpy() != 0)
    assert not (both & distinct & (fwd.numpy() != s.numpy())).any()


@pytest.mark.parametrize("kernel", [0, 2])
def test_backward_initial_state_layouts(kernel):
    # 0: automatic (the tile kernel at this size), 2: the pipelined gradient
    sgr.set_kernel_override(kernel)
    B, T, D = 3, 600, 96
    p, q, i0, fwd, gy = inputs("mingru", B, T, D, "f32", "u01_1", seed=11)
    P, Q, F, G = (t.to(DEV) for t in (p, q, fwd, gy))
    # h0 given as rows of a wider tensor, dh0 written into rows of a wider tensor
    wide = torch.zeros(B, 2 * D, device=DEV)
    wide[:, D:] = i0.to(DEV)
    dk = torch.empty_like(P)
    dhx = torch.empty_like(P)
    dwide = torch.full((B, 3 * D), 7.0, device=DEV)
    lib = _abi.lib()
    need = lib.sgr_backward_workspace_size(0, B, T, D, 0)
    ws = sgr.Workspace(need, DEV)
    code = lib.mingru_scan_backward(P.data_ptr(), Q.data_ptr(), wide[:, D:].data_ptr(), 2 * D,
                                    F.data_ptr(), G.data_ptr(), dk.data_ptr(), dhx.data_ptr(),
                                    dwide[:, D:].data_ptr(), 3 * D, B, T, D, 0, ws.ptr, ws.nbytes,
                                    torch.cuda.current_stream().cuda_stream)
    assert code == 0
    torch.cuda.synchronize()
    rk, rhx, rh0 = oracle.mingru_backward(p, q, i0, gy)
    assert channel_scaled_err(dk, rk) <= TOL_BWD["f32"]
    assert row_scaled_err(dwide[:, D:2 * D], rh0) <= TOL_BWD["f32"]
    assert bool((dwide[:, :D] == 7.0).all()) and bool((dwide[:, 2 * D:] == 7.0).all())
    # T = 0: the initial-state gradient is zero
    dh0 = torch.full((B, D), 5.0, device=DEV)
    code = lib.mingru_scan_backward(None, None, None, 0, None, None, None, None, dh0.data_ptr(), D,
                                    B, 0, D, 0, None, 0, torch.cuda.current_stream().cuda_stream)
    assert code == 0
    torch.cuda.synchronize()
    assert bool((dh0 == 0).all())


@pytest.mark.parametrize("op", ["mingru", "minmax"])
@pytest.mark.parametrize("h0_kind", [None, "rows", "vector"])
def test_autograd_wrappers(op, h0_kind):
    B, T, D = 2, 700, 64
    p, q, i0, _, gy = inputs(op, B, T, D, "f32", "u01_1", seed=21)
    init = None if h0_kind is None else (i0 if h0_kind == "rows" else i0[0].clone())
    P = p.to(DEV).requires_grad_()
    Q = q.to(DEV).requires_grad_()
    I = None if init is None else init.to(DEV).requires_grad_()
    fn = sgr.mingru_scan_fn if op == "mingru" else sgr.minmax_scan_fn
    y = fn(P, Q, I)
    (y * gy.to(DEV)).sum().backward()
    ref_init = None if init is None else (init if init.dim() == 2 else init.expand(B, D))
    rp, rq, rinit = oracle_backward(op, p, q, ref_init, gy)
    assert channel_scaled_err(P.grad, rp) <= TOL_BWD["f32"]
    assert channel_scaled_err(Q.grad, rq) <= TOL_BWD["f32"]
    if I is not None:
        want = rinit if init.dim() == 2 else rinit.sum(0)
        got = I.grad.cpu().double().numpy()
        assert row_scaled_err(got.reshape(-1, D), np.asarray(want).reshape(-1, D)) <= TOL_BWD["f32"]


def test_backward_bounded_wait_reports_timeout():
    # a chunk that never publishes: its successor's wait runs out, NaN outputs
    B, T, D = 1, 4000, 64
    p, q, i0, fwd, gy = inputs("mingru", B, T, D, "f32", None, seed=31)
    lib = _abi.lib()
    lib.sgr_set_wait_limit(64)
    lib.sgr_set_drop_publish(0)
    need = lib.sgr_backward_workspace_size(0, B, T, D, 0)
    ws = sgr.Workspace(need, DEV)
    dk, dhx, _ = sgr.mingru_scan_backward(*(t.to(DEV) for t in (p, q)), None, fwd.to(DEV), gy.to(DEV),
                                          want_dh0=False, workspace=ws)
    assert ws.status() == _abi.SGR_ERR_TIMEOUT
    assert bool(torch.isnan(dk).any())
    lib.sgr_set_drop_publish(-1)
    lib.sgr_set_wait_limit(0)
    dk, dhx, _ = sgr.mingru_scan_backward(*(t.to(DEV) for t in (p, q)), None, fwd.to(DEV), gy.to(DEV),
                                          want_dh0=False, workspace=ws)
    assert ws.status() == 0 and bool(torch.isfinite(dk).all())


def test_backward_workload_b8_t4096_d1024():
    """The gradient of the benchmark's minGRU workload, at full size, on every
    channel and row: the kernel reads the oracle's forward (rounded to fp32)
    and is compared with the oracle's gradient of the whole tensor."""
    w = WORKLOADS["mingru_b8_t4096_d1024_f32_h0"]
    K, H, H0 = generate(w, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(5)
    GY = torch.randn(K.shape, device=DEV, generator=g)
    k, hx, h0, gy = (t.cpu() for t in (K, H, H0, GY))
    Hf = torch.from_numpy(oracle.mingru_linear(k, hx, h0, threads=8)).float().to(DEV)
    dk, dhx, dh0 = sgr.mingru_scan_backward(K, H, H0, Hf, GY)
    torch.cuda.synchronize()
    rk, rhx, rh0 = oracle.mingru_backward(k, hx, h0, gy, threads=8)
    ek, ehx = channel_scaled_err(dk, rk), channel_scaled_err(dhx, rhx)
    # dL/dh0 sums signed terms over the whole sequence: its error is measured
    # against the largest |dL/dh0| of the batch row
    g0 = dh0.double().cpu().numpy()
    eh0 = float((np.abs(g0 - rh0) / np.abs(rh0).max(axis=1, keepdims=True)).max())
    print(f"{w.name} gradient: channel-scaled max error dk {ek:.3e}, dhx {ehx:.3e}, dh0 {eh0:.3e}")
    assert ek <= TOL_BWD["f32"] and ehx <= TOL_BWD["f32"]
    assert eh0 <= TOL_BWD["f32"]
