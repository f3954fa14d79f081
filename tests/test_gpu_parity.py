"""GPU parity: the CUDA library against the fp64 CPU oracle, element by element.

minGRU (page "Mingru Pytorch": log-space minGRU, batched (B, T, D), optional
carried state, token-by-token mode): max relative error <= 1e-5 with fp32 I/O,
<= 2e-2 with bf16 I/O (fp32 arithmetic).  MinMax neuron (page "MinMax
Recurrent Neural Cascades", The model, item 3): bit-exact.

Small shapes span several tiles and ragged tails in T and D and run the
oracle on every element; the benchmark's full-size workloads run in the same
launch configuration the benchmark times and are checked on a seeded sample
of channels over their full length (channels are independent), except MinMax
which is checked in full.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import scan_gated_rnns_b200 as sgr
from scan_gated_rnns_b200 import _abi
from scan_gated_rnns_b200.synth import WORKLOADS, Workload, generate

from parity import TOL, TORCH_DT, full_rel_err, rel_err

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = torch.device("cuda:0")


def to_dev(*ts):
    return [None if t is None else t.to(DEV) for t in ts]


def run(op, p, q, init, **kw):
    fn = sgr.mingru_scan if op == "mingru" else sgr.minmax_scan
    P, Q, I = to_dev(p, q, init)
    y = fn(P, Q, I, **kw)
    torch.cuda.synchronize()
    return y


def small(op, B, T, D, dtype, init, seed, k_mean=0.0):
    w = Workload("t", op, B, T, D, dtype, seed=seed, k_mean=k_mean, init=init)
    return generate(w)


SHAPES = [(2, 1024, 512), (3, 1000, 96), (1, 777, 36), (2, 300, 7), (1, 1, 1), (5, 1, 64),
          (1, 4097, 32), (2, 129, 40), (4, 63, 8), (1, 2000, 1), (2, 513, 264)]


@pytest.fixture(autouse=True)
def _reset_hooks():
    yield
    lib = _abi.lib()
    lib.sgr_set_tile_override(0, 0)
    lib.sgr_set_kernel_override(0)
    lib.sgr_set_wait_limit(0)
    lib.sgr_set_drop_publish(-1)


# (kernel, rows per thread): the tile kernel and the pipelined kernel, every R
VARIANTS = [(1, 1), (1, 2), (1, 4), (1, 8), (2, 2), (2, 4), (2, 8), (3, 2), (3, 4)]


# ------------------------------------------------------------------ minGRU

@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("init", [None, "u01_1"])
def test_mingru_matches_oracle(shape, dtype, init):
    k, hx, h0 = small("mingru", *shape, dtype, init, seed=hash(shape) % 1000)
    h = run("mingru", k, hx, h0)
    assert h.dtype == TORCH_DT[dtype] and h.shape == k.shape
    ref = oracle.mingru_linear(k, hx, h0, threads=8)
    assert rel_err(h, ref) <= TOL[dtype]
    # and against the log-space statement of the same function
    ref_log = oracle.mingru_log(k, hx, h0, threads=8)
    assert rel_err(h, ref_log) <= TOL[dtype]


@pytest.mark.parametrize("kernel,r", VARIANTS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(3, 1500, 160), (2, 3001, 384)])
def test_mingru_every_kernel_and_tile_shape(kernel, r, dtype, shape):
    sgr.set_kernel_override(kernel)
    sgr.set_tile_override(0, r)
    k, hx, h0 = small("mingru", *shape, dtype, "u01_1", seed=kernel * 10 + r)
    pl = _abi.plan(0, *shape, 0 if dtype == "f32" else 1, True)
    assert pl["kernel"] == kernel and pl["n_chunks"] > 1
    h = run("mingru", k, hx, h0)
    assert rel_err(h, oracle.mingru_linear(k, hx, h0, threads=8)) <= TOL[dtype]


def test_mingru_gate_closed_forms():
    # z = 1 (k = +inf): h_t = g(hx_t); z = 0 (k = -inf): h_t = h_0 exactly
    B, T, D = 2, 700, 64
    g = torch.Generator().manual_seed(5)
    hx = torch.randn(B, T, D, generator=g) * 3
    h0 = torch.rand(B, D, generator=g) * 0.9 + 0.1
    h = run("mingru", torch.full((B, T, D), math.inf), hx, h0)
    want = torch.where(hx >= 0, hx.double() + 0.5, torch.sigmoid(hx.double()))
    assert rel_err(h, want.numpy()) <= TOL["f32"]
    h = run("mingru", torch.full((B, T, D), -math.inf), hx, h0)
    assert torch.equal(h.cpu(), h0[:, None, :].expand(B, T, D))
    h = run("mingru", torch.full((B, T, D), -math.inf), hx, None)
    assert torch.equal(h.cpu(), torch.zeros(B, T, D))


def test_mingru_initial_state_layouts():
    B, T, D = 3, 600, 96
    k, hx, h0 = small("mingru", B, T, D, "f32", "u01_1", seed=11)
    # (D,) broadcast to every batch row
    v = h0[1]
    h = run("mingru", k, hx, v)
    assert rel_err(h, oracle.mingru_linear(k, hx, v.expand(B, D).contiguous())) <= TOL["f32"]
    # rows of a wider tensor (batch stride 2 D)
    wide = torch.rand(B, 2 * D) + 0.1
    h = run("mingru", k, hx, wide[:, D:])
    assert rel_err(h, oracle.mingru_linear(k, hx, wide[:, D:].contiguous())) <= TOL["f32"]


def test_mingru_misaligned_operands_take_scalar_path():
    B, T, D = 2, 400, 64
    k, hx, h0 = small("mingru", B, T, D, "f32", "u01_1", seed=12)
    n = B * T * D
    kb = torch.empty(n + 1, device=DEV)
    hb = torch.empty(n + 1, device=DEV)
    kb[1:].copy_(k.reshape(-1).to(DEV))
    hb[1:].copy_(hx.reshape(-1).to(DEV))
    K, H = kb[1:].view(B, T, D), hb[1:].view(B, T, D)
    assert _abi.plan(0, B, T, D, 0, K.data_ptr() % 16 == 0)["vector_path"] == 0
    y = sgr.mingru_scan(K, H, h0.to(DEV))
    assert rel_err(y, oracle.mingru_linear(k, hx, h0)) <= TOL["f32"]


def test_empty_shapes():
    for shp in [(0, 5, 8), (2, 0, 8), (2, 5, 0)]:
        z = torch.zeros(shp, device=DEV)
        assert sgr.mingru_scan(z, z).shape == shp
        assert sgr.minmax_scan(z, z).shape == shp


def test_output_overlapping_input_is_rejected():
    k = torch.randn(2, 64, 32, device=DEV)
    hx = torch.randn(2, 64, 32, device=DEV)
    with pytest.raises(sgr.ScanError) as e:
        sgr.mingru_scan(k, hx, out=k)
    assert e.value.code == _abi.SGR_ERR_INVALID_ARG


def test_workspace_reused_across_shapes_and_ops():
    # one explicit workspace, several calls of different shapes: the per-launch
    # epoch must keep every chunk from reading a summary another launch left
    ws = sgr.Workspace(sgr.workspace_size("mingru", 4, 5000, 96, torch.float32), DEV)
    cases = [("mingru", (2, 3000, 64)), ("minmax", (4, 5000, 96)), ("mingru", (4, 5000, 96)),
             ("mingru", (2, 3000, 64)), ("minmax", (1, 4000, 32))]
    for i, (op, shp) in enumerate(cases):
        p, q, init = small(op, *shp, "f32", "u01_1", seed=40 + i)
        y = run(op, p, q, init, workspace=ws)
        if op == "mingru":
            assert rel_err(y, oracle.mingru_linear(p, q, init, threads=8)) <= TOL["f32"]
        else:
            assert np.array_equal(y.cpu().double().numpy(), oracle.minmax(p, q, init, threads=8))
    assert ws.status() == _abi.SGR_OK


def test_graph_capture_replays():
    B, T, D = 2, 3000, 64
    k0, hx0, h00 = small("mingru", B, T, D, "f32", "u01_1", seed=21)
    K, H, H0 = to_dev(k0, hx0, h00)
    out = torch.empty_like(K)
    ws = sgr.Workspace(sgr.workspace_size("mingru", B, T, D, torch.float32), DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        sgr.mingru_scan(K, H, H0, out=out, workspace=ws)      # warm-up outside the graph
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            sgr.mingru_scan(K, H, H0, out=out, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    for seed in (22, 23, 24):
        k, hx, h0 = small("mingru", B, T, D, "f32", "u01_1", seed=seed)
        K.copy_(k.to(DEV)); H.copy_(hx.to(DEV)); H0.copy_(h0.to(DEV))
        graph.replay()
        torch.cuda.synchronize()
        assert rel_err(out, oracle.mingru_linear(k, hx, h0, threads=8)) <= TOL["f32"]
        # an eager call between replays on the same workspace
        y = sgr.mingru_scan(K, H, H0, workspace=ws)
        torch.cuda.synchronize()
        assert rel_err(y, oracle.mingru_linear(k, hx, h0, threads=8)) <= TOL["f32"]


@pytest.mark.parametrize("kernel,D", [(1, 64), (2, 64), (3, 64)])
def test_bounded_wait_reports_timeout(kernel, D):
    # chunk 0 of channel tile 0 skips publishing its state: the next chunk of the
    # same channels waits until the poll limit, records the timeout and writes
    # NaN; every other channel tile is unaffected
    B, T = 1, 2048
    k, hx, h0 = small("mingru", B, T, D, "f32", "u01_1", seed=31)
    sgr.set_kernel_override(kernel)
    sgr.set_tile_override(0, 1 if kernel == 1 else 2)
    pl = _abi.plan(0, B, T, D, 0, True)
    assert pl["kernel"] == kernel and pl["n_chunks"] > 2 and pl["n_chains"] == 2
    ws = sgr.Workspace(pl["workspace_bytes"], DEV)
    lib = _abi.lib()
    lib.sgr_set_wait_limit(2000)
    lib.sgr_set_drop_publish(0)
    y = run("mingru", k, hx, h0, workspace=ws)
    assert ws.status(clear=True) == _abi.SGR_ERR_TIMEOUT
    TR, TC = pl["tile_rows"], pl["tile_channels"]
    ref = oracle.mingru_linear(k, hx, h0)
    yc = y.cpu().double().numpy()
    assert rel_err(yc[:, :TR, :TC], ref[:, :TR, :TC]) <= TOL["f32"]   # chunk 0 itself is fine
    assert np.isnan(yc[:, TR:, :TC]).all()                              # its successors are NaN
    assert rel_err(yc[:, :, TC:], ref[:, :, TC:]) <= TOL["f32"]         # other channels fine
    # with the hooks cleared the same workspace works and reports no error
    lib.sgr_set_drop_publish(-1)
    lib.sgr_set_wait_limit(0)
    y = run("mingru", k, hx, h0, workspace=ws)
    assert ws.status() == _abi.SGR_OK
    assert rel_err(y, ref) <= TOL["f32"]


# ------------------------------------------------------------------ step

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_step_matches_oracle_and_scan(dtype):
    B, T, D = 4, 40, 72
    k, hx, h0 = small("mingru", B, T, D, dtype, "u01_1", seed=51)
    K, H, H0 = to_dev(k, hx, h0)
    state = H0.clone()
    outs = []
    for t in range(T):
        sgr.mingru_step(K[:, t, :], H[:, t, :], state, out=state)   # strided rows, in place
        outs.append(state.clone())
    torch.cuda.synchronize()
    got = torch.stack(outs, dim=1)
    assert rel_err(got, oracle.mingru_linear(k, hx, h0)) <= TOL[dtype]
    # no initial state
    h1 = sgr.mingru_step(K[:, 0, :], H[:, 0, :])
    torch.cuda.synchronize()
    assert rel_err(h1, oracle.mingru_step(k[:, 0, :], hx[:, 0, :])) <= TOL[dtype]


# ------------------------------------------------------------------ MinMax

def exact(y: torch.Tensor, ref: np.ndarray) -> bool:
    """Bitwise equality in the I/O dtype (the oracle's values are inputs)."""
    want = torch.from_numpy(ref).to(y.dtype)
    return torch.equal(y.cpu(), want)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("init", [None, "u01_1"])
def test_minmax_bit_exact(shape, dtype, init):
    r, s, x0 = small("minmax", *shape, dtype, init, seed=hash(shape) % 1000 + 7)
    x = run("minmax", r, s, x0)
    assert exact(x, oracle.minmax(r, s, x0, threads=8))


@pytest.mark.parametrize("kernel,rr", VARIANTS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_minmax_every_kernel_and_tile_shape(kernel, rr, dtype):
    sgr.set_kernel_override(kernel)
    sgr.set_tile_override(0, rr)
    r, s, x0 = small("minmax", 3, 2500, 160, dtype, "u01_1", seed=kernel + rr)
    assert exact(run("minmax", r, s, x0), oracle.minmax(r, s, x0, threads=8))


def test_minmax_special_values():
    # infinities and repeated values (ties) on a small grid of values
    g = torch.Generator().manual_seed(3)
    vals = torch.tensor([-math.inf, -2.0, -0.5, 0.5, 1.0, 3.0, math.inf])
    r = vals[torch.randint(0, 7, (2, 3000, 40), generator=g)]
    s = vals[torch.randint(0, 7, (2, 3000, 40), generator=g)]
    x0 = vals[torch.randint(0, 7, (2, 40), generator=g)]
    assert exact(run("minmax", r, s, x0), oracle.minmax(r, s, x0, threads=8))


# ------------------------------------------------- full-size workloads

def test_workload_mingru_b2_t1024_d512():
    w = WORKLOADS["mingru_b2_t1024_d512_f32"]
    k, hx, h0 = generate(w, device=DEV)
    h = sgr.mingru_scan(k, hx, h0)
    torch.cuda.synchronize()
    err = rel_err(h, oracle.mingru_linear(k, hx, h0, threads=8))
    print(f"{w.name}: max relative error {err:.3e} (bar {TOL['f32']:.0e})")
    assert err <= TOL["f32"]


def test_workload_mingru_b8_t4096_d1024_and_steps():
    w = WORKLOADS["mingru_b8_t4096_d1024_f32_h0"]
    K, H, H0 = generate(w, device=DEV)
    full = sgr.mingru_scan(K, H, H0)
    torch.cuda.synchronize()
    err = full_rel_err("mingru", K, H, H0, full)           # every channel and row
    print(f"{w.name}: max relative error {err:.3e} (bar {TOL['f32']:.0e})")
    assert err <= TOL["f32"]
    # first 4000 tokens in parallel, then 96 single-token steps
    pre = sgr.mingru_scan(K[:, :4000].contiguous(), H[:, :4000].contiguous(), H0)
    state = pre[:, -1, :].clone()
    tail = []
    for t in range(4000, 4096):
        sgr.mingru_step(K[:, t, :], H[:, t, :], state, out=state)
        tail.append(state.clone())
    torch.cuda.synchronize()
    stitched = torch.cat([pre, torch.stack(tail, dim=1)], dim=1)
    assert rel_err(stitched, full.double().cpu().numpy()) <= TOL["f32"]
    err = full_rel_err("mingru", K, H, H0, stitched)
    print(f"{w.name} (4000 scanned + 96 steps): max relative error {err:.3e}")
    assert err <= TOL["f32"]


def test_workload_minmax_b4_t8192_d768():
    w = WORKLOADS["minmax_b4_t8192_d768_f32"]
    r, s, x0 = generate(w, device=DEV)
    x = sgr.minmax_scan(r, s, x0)
    torch.cuda.synchronize()
    assert exact(x, oracle.minmax(r, s, x0, threads=8))


def test_workload_long_sequence():
    w = WORKLOADS["mingru_b1_t131072_d512_f32_h0"]
    k, hx, h0 = generate(w, device=DEV)
    h = sgr.mingru_scan(k, hx, h0)
    torch.cuda.synchronize()
    err = full_rel_err("mingru", k, hx, h0, h)             # every channel and row
    print(f"{w.name}: max relative error {err:.3e} (bar {TOL['f32']:.0e})")
    assert err <= TOL["f32"]


def test_workload_bf16_throughput_shape():
    w = WORKLOADS["mingru_b16_t2048_d4096_bf16_h0"]
    k, hx, h0 = generate(w, device=DEV)
    h = sgr.mingru_scan(k, hx, h0)
    torch.cuda.synchronize()
    err = full_rel_err("mingru", k, hx, h0, h)             # every channel and row
    print(f"{w.name}: max relative error {err:.3e} (bar {TOL['bf16']:.0e})")
    assert err <= TOL["bf16"]
