"""GPU parity of the host-buffer scans (mingru_scan_host, minmax_scan_host)
against the fp64 CPU oracle.

The operands live in host memory; the library cuts T into slices, each
started from the previous slice's last output row, so the bars are those of
the device scans: minGRU (page "Mingru Pytorch", log-space minGRU with an
optional carried state) max relative error <= 1e-5 fp32, <= 2e-2 bf16; MinMax
neuron (page "MinMax Recurrent Neural Cascades", The model, item 3) bit-exact.
Slice counts cover one slice, ragged last slices, one row per slice and the
automatic choice.
"""
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


def small(op, B, T, D, dtype, init, seed):
    return generate(Workload("t", op, B, T, D, dtype, seed=seed, init=init))


def pinned(*ts):
    return [None if t is None else t.pin_memory() for t in ts]


SHAPES = [(2, 1024, 512), (3, 1000, 96), (1, 777, 36), (2, 300, 7), (5, 1, 64), (4, 63, 8)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("chunks", [0, 1, 3, 10**6])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("init", [None, "u01_1"])
def test_mingru_host_matches_oracle(shape, chunks, dtype, init):
    k, hx, h0 = pinned(*small("mingru", *shape, dtype, init, seed=sum(shape) + chunks % 97))
    h = sgr.mingru_scan_host(k, hx, h0, chunks=chunks)
    assert not h.is_cuda and h.dtype == TORCH_DT[dtype] and h.shape == k.shape
    assert h.is_pinned()
    assert rel_err(h, oracle.mingru_linear(k, hx, h0, threads=8)) <= TOL[dtype]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("chunks", [0, 2, 7])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("init", [None, "u01_1"])
def test_minmax_host_bit_exact(shape, chunks, dtype, init):
    r, s, x0 = pinned(*small("minmax", *shape, dtype, init, seed=sum(shape) + 5))
    x = sgr.minmax_scan_host(r, s, x0, chunks=chunks)
    assert torch.equal(x.to(torch.float64), torch.from_numpy(oracle.minmax(r, s, x0, threads=8)))
    # and bit-identical to the device scan of the same data
    y = sgr.minmax_scan(r.to(DEV), s.to(DEV), None if x0 is None else x0.to(DEV))
    assert torch.equal(x, y.cpu())


def test_host_initial_state_layouts_and_pageable_memory():
    B, T, D = 3, 900, 96
    k, hx, h0 = small("mingru", B, T, D, "f32", "u01_1", seed=21)   # pageable
    v = h0[1].clone()
    h = sgr.mingru_scan_host(k, hx, v, chunks=4)
    assert not h.is_pinned()
    assert rel_err(h, oracle.mingru_linear(k, hx, v.expand(B, D).contiguous())) <= TOL["f32"]
    wide = torch.rand(B, 2 * D, generator=torch.Generator().manual_seed(2)) + 0.1
    h = sgr.mingru_scan_host(k, hx, wide[:, D:], chunks=5)
    assert rel_err(h, oracle.mingru_linear(k, hx, wide[:, D:].contiguous())) <= TOL["f32"]


def test_host_operands_need_no_alignment():
    B, T, D = 2, 500, 37
    k, hx, h0 = small("mingru", B, T, D, "f32", "u01_1", seed=22)
    n = B * T * D
    kb, hb = torch.empty(n + 1).pin_memory(), torch.empty(n + 1).pin_memory()
    kb[1:].copy_(k.reshape(-1))
    hb[1:].copy_(hx.reshape(-1))
    K, H = kb[1:].view(B, T, D), hb[1:].view(B, T, D)
    assert K.data_ptr() % 16 != 0
    h = sgr.mingru_scan_host(K, H, h0, chunks=3)
    assert rel_err(h, oracle.mingru_linear(k, hx, h0)) <= TOL["f32"]


def test_back_to_back_calls_share_staging():
    # two enqueued calls on one stream and one staging buffer, one sync
    a = pinned(*small("mingru", 2, 2000, 256, "f32", "u01_1", seed=23))
    b = pinned(*small("mingru", 2, 2000, 256, "f32", None, seed=24))
    ha = sgr.mingru_scan_host(*a, chunks=6, blocking=False)
    hb = sgr.mingru_scan_host(*b, chunks=6, blocking=False)
    torch.cuda.current_stream().synchronize()
    assert rel_err(ha, oracle.mingru_linear(*a, threads=8)) <= TOL["f32"]
    assert rel_err(hb, oracle.mingru_linear(*b, threads=8)) <= TOL["f32"]


def test_host_entry_rejects_bad_arguments():
    lib = _abi.lib()
    B, T, D = 2, 64, 32
    k, hx, _ = pinned(*small("mingru", B, T, D, "f32", None, seed=25))
    out = torch.empty_like(k).pin_memory()
    need = sgr.staging_size("mingru", B, T, D, torch.float32)
    st = torch.empty(need, dtype=torch.uint8, device=DEV)
    s = torch.cuda.current_stream().cuda_stream

    def call(p, q, o, staging=st.data_ptr(), nbytes=need, chunks=0):
        return lib.mingru_scan_host(p, q, None, 0, o, B, T, D, _abi.SGR_F32, chunks, staging,
                                    nbytes, s)

    kd = k.to(DEV)
    assert call(kd.data_ptr(), hx.data_ptr(), out.data_ptr()) == _abi.SGR_ERR_INVALID_ARG
    assert call(k.data_ptr(), hx.data_ptr(), k.data_ptr()) == _abi.SGR_ERR_INVALID_ARG
    assert call(k.data_ptr(), hx.data_ptr(), out.data_ptr(), chunks=-1) == _abi.SGR_ERR_INVALID_ARG
    assert call(k.data_ptr(), hx.data_ptr(), out.data_ptr(), nbytes=need - 1) == _abi.SGR_ERR_WORKSPACE
    assert call(k.data_ptr(), hx.data_ptr(), out.data_ptr(), staging=None) == _abi.SGR_ERR_WORKSPACE
    assert call(k.data_ptr(), hx.data_ptr(), out.data_ptr()) == _abi.SGR_OK
    torch.cuda.synchronize()
    assert rel_err(out, oracle.mingru_linear(k, hx)) <= TOL["f32"]


def test_host_workload_b8_t4096_d1024():
    """The end-to-end configuration the benchmark times (automatic slices)."""
    w = WORKLOADS["mingru_b8_t4096_d1024_f32_h0"]
    K, H, H0 = generate(w, device=DEV)
    k, hx, h0 = pinned(K.cpu(), H.cpu(), H0.cpu())
    h = sgr.mingru_scan_host(k, hx, h0)
    err = full_rel_err("mingru", k, hx, h0, h)             # every channel and row
    print(f"{w.name} from host memory: max relative error {err:.3e}")
    assert err <= TOL["f32"]
    full = sgr.mingru_scan(K, H, H0)
    torch.cuda.synchronize()
    assert rel_err(h, full.cpu().double().numpy()) <= 2e-5
