"""GPU parity of the split-time-axis path: slice summaries
(sgr_scan_summary), their combination into a slice's incoming state
(sgr_combine_summaries), and a whole sequence scanned as R slices on one GPU
(the ranks emulated in one process, the all-gather replaced by stacking the
pairs), against the fp64 oracle over the whole sequence.

Summaries are pinned through the oracle's forward: a minGRU slice maps a
starting state x to A x + B, so B = h_end(0) and A = h_end(1) - h_end(0); a
MinMax slice maps x to max(min(x, U), L), checked by applying the pair to
several starting states including +-inf (exactly).
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import scan_gated_rnns_b200 as sgr
from scan_gated_rnns_b200 import sharded
from scan_gated_rnns_b200.synth import Workload, generate

from parity import TOL, TORCH_DT, rel_err

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = torch.device("cuda:0")


def data(op, B, T, D, dtype, init, seed):
    return generate(Workload("t", op, B, T, D, dtype, seed=seed, init=init))


@pytest.mark.parametrize("shape", [(2, 1000, 96), (3, 4097, 40), (1, 1, 8), (2, 300, 7), (4, 63, 264)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_mingru_summary_matches_oracle(shape, dtype):
    k, hx, _ = data("mingru", *shape, dtype, None, seed=sum(shape) % 71)
    pairs = sharded.scan_summary("mingru", k.to(DEV), hx.to(DEV)).cpu().double().numpy()
    B, T, D = shape
    h_zero = oracle.mingru_linear(k, hx, np.zeros((B, D)))[:, -1]
    h_one = oracle.mingru_linear(k, hx, np.ones((B, D)))[:, -1]
    tol = 1e-5 if dtype == "f32" else 1e-5   # fp32 arithmetic on exact bf16 inputs either way
    np.testing.assert_allclose(pairs[..., 1], h_zero, rtol=tol, atol=1e-30)
    # A is a product of T gates, each rounded in fp32: its relative error grows
    # with T (about sqrt(T) ulps typically, T ulps at worst), hence 1e-4 here
    np.testing.assert_allclose(pairs[..., 0], h_one - h_zero, rtol=1e-4, atol=1e-7)


@pytest.mark.parametrize("shape", [(2, 1000, 96), (3, 4097, 40), (1, 1, 8), (2, 300, 7)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_minmax_summary_is_exact(shape, dtype):
    r, s, _ = data("minmax", *shape, dtype, None, seed=sum(shape) % 73)
    pairs = sharded.scan_summary("minmax", r.to(DEV), s.to(DEV)).cpu().double().numpy()
    B, T, D = shape
    for x0 in (np.inf, -np.inf, 0.0, 0.7, -1.3):
        start = np.full((B, D), x0)
        want = oracle.minmax(r, s, start)[:, -1]
        got = np.maximum(np.minimum(start, pairs[..., 0]), pairs[..., 1])
        np.testing.assert_array_equal(got, want)


def test_empty_slice_summary_is_identity():
    k = torch.empty(2, 0, 8, device=DEV)
    for op, want in (("mingru", (1.0, 0.0)), ("minmax", (np.inf, -np.inf))):
        pairs = sharded.scan_summary(op, k, k).cpu().numpy()
        assert np.all(pairs[..., 0] == want[0]) and np.all(pairs[..., 1] == want[1])


@pytest.mark.parametrize("op", ["mingru", "minmax"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("cuts", [(0, 1000, 2500, 4096), (0, 0, 4096), (0, 1, 2, 3000, 4096)])
def test_sequence_split_into_slices_on_one_gpu(op, dtype, cuts):
    B, T, D = 2, cuts[-1], 160
    p, q, init = data(op, B, T, D, dtype, "u01_1", seed=len(cuts))
    P, Q, I = p.to(DEV), q.to(DEV), init.to(DEV)
    slices = list(zip(cuts[:-1], cuts[1:]))
    pairs = torch.stack([sharded.scan_summary(op, P[:, a:b].contiguous(), Q[:, a:b].contiguous())
                         for a, b in slices], 0).contiguous()
    outs = []
    for rank, (a, b) in enumerate(slices):
        h_in = sharded.combine_summaries(op, pairs, rank, I, P.dtype)
        fn = sgr.mingru_scan if op == "mingru" else sgr.minmax_scan
        outs.append(fn(P[:, a:b].contiguous(), Q[:, a:b].contiguous(), h_in))
    got = torch.cat(outs, 1)
    torch.cuda.synchronize()
    if op == "mingru":
        assert rel_err(got, oracle.mingru_linear(p, q, init, threads=8)) <= TOL[dtype]
    else:
        assert torch.equal(got.cpu().double(), torch.from_numpy(oracle.minmax(p, q, init, threads=8)))


def test_time_sharded_scan_through_nccl_single_rank():
    import torch.distributed as dist
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=DEV)
    try:
        k, hx, h0 = data("mingru", 2, 3000, 96, "f32", "u01_1", seed=9)
        got = sharded.time_sharded_scan("mingru", k.to(DEV), hx.to(DEV), h0.to(DEV))
        want = sgr.mingru_scan(k.to(DEV), hx.to(DEV), h0.to(DEV))
        torch.cuda.synchronize()
        assert torch.allclose(got, want, rtol=1e-6, atol=0)
    finally:
        dist.destroy_process_group()
