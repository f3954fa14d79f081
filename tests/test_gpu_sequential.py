"""GPU parity of the channel-sequential scan kernel against the fp64 oracle.

The kernel gives each warp one group of 32 channels of one batch row and
walks the whole sequence in order; the library picks it when the channel
groups alone fill the GPU.  Here it is
forced (kernel override 4) on small ragged shapes -- T not a multiple of the
16-row slots, D not a multiple of the channel group, T = 1, several ring
wraps -- for every operation it serves: minGRU (page "Mingru Pytorch":
max relative error <= 1e-5 fp32, <= 2e-2 bf16), the MinMax neuron (page
"MinMax Recurrent Neural Cascades", The model, item 3: bit-exact) and the
time-decayed minGRU (page "Your first delta model", Step 5, read for a
vector state).  Shapes that select it automatically are checked too, and the
bf16 throughput workload runs it at full size in the benchmark's launch.
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
SEQ = _abi.KERNEL_SEQUENTIAL
# 7, 8: two channels per lane (two or four warps per group), bf16 only (fp32
# takes kind 6 under those overrides)
SEQ_KINDS = (_abi.KERNEL_SEQUENTIAL, _abi.KERNEL_SEQUENTIAL_SPLIT, _abi.KERNEL_SEQUENTIAL_PAIR,
             _abi.KERNEL_SEQUENTIAL_PAIR2, _abi.KERNEL_SEQUENTIAL_QUAD)
WIDE_KINDS = (_abi.KERNEL_SEQUENTIAL_PAIR2, _abi.KERNEL_SEQUENTIAL_QUAD)


@pytest.fixture(autouse=True)
def _reset_hooks():
    yield
    lib = _abi.lib()
    lib.sgr_set_tile_override(0, 0)
    lib.sgr_set_kernel_override(0)


def small(op, B, T, D, dtype, init, seed, k_mean=0.0):
    return generate(Workload("t", op, B, T, D, dtype, seed=seed, k_mean=k_mean, init=init))


def dev(*ts):
    return [None if t is None else t.to(DEV) for t in ts]


def exact(y: torch.Tensor, ref: np.ndarray) -> bool:
    return torch.equal(y.cpu(), torch.from_numpy(ref).to(y.dtype))


def plan(B, T, D, dtype):
    return _abi.plan(0, B, T, D, 0 if dtype == "f32" else 1, True)


# T: one row, under a slot, ragged slots, many ring wraps; D: partial groups
SHAPES = [(2, 1, 64), (3, 17, 40), (2, 300, 96), (1, 1000, 200), (4, 129, 8), (2, 2049, 136)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("init", [None, "u01_1"])
@pytest.mark.parametrize("kind", SEQ_KINDS)
def test_mingru_sequential_matches_oracle(shape, dtype, init, kind):
    sgr.set_kernel_override(kind)
    want = _abi.KERNEL_SEQUENTIAL_PAIR if (kind in WIDE_KINDS and dtype == "f32") else kind
    assert plan(*shape, dtype)["kernel"] == want
    k, hx, h0 = small("mingru", *shape, dtype, init, seed=sum(shape) % 97)
    h = sgr.mingru_scan(*dev(k, hx, h0))
    torch.cuda.synchronize()
    assert h.dtype == TORCH_DT[dtype] and h.shape == k.shape
    assert rel_err(h, oracle.mingru_linear(k, hx, h0, threads=8)) <= TOL[dtype]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("init", [None, "u01_1"])
@pytest.mark.parametrize("kind", SEQ_KINDS)
def test_minmax_sequential_bit_exact(shape, dtype, init, kind):
    sgr.set_kernel_override(kind)
    r, s, x0 = small("minmax", *shape, dtype, init, seed=sum(shape) % 89 + 3)
    x = sgr.minmax_scan(*dev(r, s, x0))
    torch.cuda.synchronize()
    assert exact(x, oracle.minmax(r, s, x0, threads=8))


@pytest.mark.parametrize("kind", SEQ_KINDS)
def test_minmax_sequential_special_values(kind):
    sgr.set_kernel_override(kind)
    g = torch.Generator().manual_seed(3)
    vals = torch.tensor([-math.inf, -2.0, -0.5, 0.5, 1.0, 3.0, math.inf])
    r = vals[torch.randint(0, 7, (2, 777, 96), generator=g)]
    s = vals[torch.randint(0, 7, (2, 777, 96), generator=g)]
    x0 = vals[torch.randint(0, 7, (2, 96), generator=g)]
    x = sgr.minmax_scan(*dev(r, s, x0))
    torch.cuda.synchronize()
    assert exact(x, oracle.minmax(r, s, x0, threads=8))


@pytest.mark.parametrize("kind", SEQ_KINDS)
def test_mingru_sequential_gate_closed_forms(kind):
    # z = 1 (k = +inf): h_t = g(hx_t); z = 0 (k = -inf): h_t = h_0 exactly
    sgr.set_kernel_override(kind)
    B, T, D = 2, 333, 64
    g = torch.Generator().manual_seed(5)
    hx = torch.randn(B, T, D, generator=g) * 3
    h0 = torch.rand(B, D, generator=g) * 0.9 + 0.1
    h = sgr.mingru_scan(*dev(torch.full((B, T, D), math.inf), hx, h0))
    torch.cuda.synchronize()
    want = torch.where(hx >= 0, hx.double() + 0.5, torch.sigmoid(hx.double()))
    assert rel_err(h, want.numpy()) <= TOL["f32"]
    h = sgr.mingru_scan(*dev(torch.full((B, T, D), -math.inf), hx, h0))
    torch.cuda.synchronize()
    assert torch.equal(h.cpu(), h0[:, None, :].expand(B, T, D))


@pytest.mark.parametrize("kind", SEQ_KINDS)
def test_mingru_sequential_initial_state_layouts(kind):
    sgr.set_kernel_override(kind)
    B, T, D = 3, 200, 96
    k, hx, h0 = small("mingru", B, T, D, "f32", "u01_1", seed=11)
    K, H = dev(k, hx)
    # one D-vector broadcast to every batch row (stride 0)
    h = sgr.mingru_scan(K, H, h0[1].to(DEV))
    torch.cuda.synchronize()
    assert rel_err(h, oracle.mingru_linear(k, hx, h0[1].expand(B, D).contiguous())) <= TOL["f32"]
    # rows of a wider tensor (batch stride 2 D)
    wide = torch.rand(B, 2 * D) + 0.1
    h = sgr.mingru_scan(K, H, wide.to(DEV)[:, D:])
    torch.cuda.synchronize()
    assert rel_err(h, oracle.mingru_linear(k, hx, wide[:, D:].contiguous())) <= TOL["f32"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("log1p_delta", [False, True])
@pytest.mark.parametrize("kind", SEQ_KINDS)
def test_decay_sequential_matches_oracle(dtype, log1p_delta, kind):
    sgr.set_kernel_override(kind)
    B, T, D = 3, 500, 136
    k, hx, h0 = small("mingru", B, T, D, dtype, "u01_1", seed=61)
    g = torch.Generator().manual_seed(62)
    dt = torch.empty(B, T).exponential_(1.0 / (20.0 if log1p_delta else 0.5), generator=g)
    dt[:, T // 2] = 3e4                                   # wipes the state
    lam = torch.rand(D, generator=g) * 2.0
    h = sgr.mingru_scan_decay(*dev(k, hx, h0, dt, lam), log1p_delta)
    torch.cuda.synchronize()
    assert rel_err(h, oracle.mingru_decay(k, hx, h0, dt, lam, log1p_delta)) <= TOL[dtype]


@pytest.mark.parametrize("dtype,shape", [("bf16", (16, 40, 4096)), ("f32", (40, 50, 768)),
                                         ("bf16", (64, 33, 1024))])
def test_wide_batches_select_it_automatically(dtype, shape):
    pl = plan(*shape, dtype)
    assert pl["kernel"] in SEQ_KINDS and pl["workspace_bytes"] == 256    # the header: status word
    k, hx, h0 = small("mingru", *shape, dtype, "u01_1", seed=71)
    h = sgr.mingru_scan(*dev(k, hx, h0))
    torch.cuda.synchronize()
    assert rel_err(h, oracle.mingru_linear(k, hx, h0, threads=8)) <= TOL[dtype]
    # and the same call with a workspace reports no error in its status word
    ws = sgr.Workspace(256, DEV)
    h2 = sgr.mingru_scan(*dev(k, hx, h0), workspace=ws)
    assert ws.status() == _abi.SGR_OK
    assert torch.equal(h2, h)


def test_misaligned_rows_do_not_take_it():
    # D * 4 bytes not a multiple of 16: the scalar chunked variant runs
    sgr.set_kernel_override(SEQ)
    assert plan(4, 100, 6, "f32")["kernel"] == _abi.KERNEL_TILE
    k, hx, h0 = small("mingru", 4, 100, 6, "f32", "u01_1", seed=72)
    h = sgr.mingru_scan(*dev(k, hx, h0))
    torch.cuda.synchronize()
    assert rel_err(h, oracle.mingru_linear(k, hx, h0)) <= TOL["f32"]


@pytest.mark.parametrize("kind", SEQ_KINDS)
def test_sequential_graph_capture_replays(kind):
    sgr.set_kernel_override(kind)
    B, T, D = 2, 300, 128
    k0, hx0, h00 = small("mingru", B, T, D, "bf16", "u01_1", seed=81)
    K, H, H0 = dev(k0, hx0, h00)
    out = torch.empty_like(K)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        sgr.mingru_scan(K, H, H0, out=out)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            sgr.mingru_scan(K, H, H0, out=out)
    torch.cuda.current_stream().wait_stream(s)
    for seed in (82, 83):
        k, hx, h0 = small("mingru", B, T, D, "bf16", "u01_1", seed=seed)
        K.copy_(k.to(DEV)); H.copy_(hx.to(DEV)); H0.copy_(h0.to(DEV))
        graph.replay()
        torch.cuda.synchronize()
        assert rel_err(out, oracle.mingru_linear(k, hx, h0, threads=8)) <= TOL["bf16"]


@pytest.mark.parametrize("kind,label", [(_abi.KERNEL_PIPELINED, "the chunked kernel"),
                                        (_abi.KERNEL_SEQUENTIAL_PAIR2, "64-channel warp pairs"),
                                        (_abi.KERNEL_SEQUENTIAL_QUAD, "64-channel groups of four warps")])
def test_bf16_workload_other_kernels_still_match(kind, label):
    # the full-size bf16 workload through the chunked pipelined kernel and the
    # two-channels-per-lane kernel (the automatic choice there is the two-warp
    # channel-sequential kernel with 32-channel groups)
    w = WORKLOADS["mingru_b16_t2048_d4096_bf16_h0"]
    assert plan(w.B, w.T, w.D, "bf16")["kernel"] == _abi.KERNEL_SEQUENTIAL_PAIR
    sgr.set_kernel_override(kind)
    assert plan(w.B, w.T, w.D, "bf16")["kernel"] == kind
    k, hx, h0 = generate(w, device=DEV)
    h = sgr.mingru_scan(k, hx, h0)
    torch.cuda.synchronize()
    err = full_rel_err("mingru", k, hx, h0, h)             # every channel and row
    print(f"{w.name} through {label}: max relative error {err:.3e}")
    assert err <= TOL["bf16"]


@pytest.mark.parametrize("dtype,shape,forced", [
    ("bf16", (128, 20, 4096), None),    # 8192 groups of 64 channels (kernel 7): several waves
    ("bf16", (128, 20, 4096), SEQ),     # 16384 warps: ~111 per SM, several waves
    ("f32", (1, 70000, 32), SEQ),       # one warp, 4375 slots: every ring slot reused many times
    ("f32", (1, 70001, 32), _abi.KERNEL_SEQUENTIAL_PAIR),    # two warps, 2188 slots, a ragged last one
    ("bf16", (2, 30001, 48), _abi.KERNEL_SEQUENTIAL_SPLIT),  # half-warps, partial channel groups
])
def test_sequential_many_waves_and_long_sequences(dtype, shape, forced):
    if forced:
        sgr.set_kernel_override(forced)
    pl = plan(*shape, dtype)
    assert pl["kernel"] == (forced or _abi.KERNEL_SEQUENTIAL_PAIR2)
    k, hx, h0 = small("mingru", *shape, dtype, "u01_1", seed=101)
    h = sgr.mingru_scan(*dev(k, hx, h0))
    r, s, x0 = small("minmax", *shape, dtype, "u01_1", seed=102)
    x = sgr.minmax_scan(*dev(r, s, x0))
    torch.cuda.synchronize()
    assert rel_err(h, oracle.mingru_linear(k, hx, h0, threads=8)) <= TOL[dtype]
    assert exact(x, oracle.minmax(r, s, x0, threads=8))
