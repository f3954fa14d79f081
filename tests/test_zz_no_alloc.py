"""mingru_scan_noalloc: the scan for callers that cannot allocate device memory
where they run it (a runtime plugin whose enqueue step must not allocate, a
fixed device-memory plan, code running under stream capture).  Its scratch is
a fixed array inside the library instead of a caller-provided workspace.

Checked through the C ABI, on two calls in a row (the second reuses the array
the first left behind), against the CPU oracle within the fp32 parity
tolerance of the other tests and against mingru_scan on the same inputs: once
on the persistent kernel's shape (hand-off words in the array) and once on
unaligned rows, where one block per chunk takes its chunk number from the
ticket counter in the array.  A shape whose scratch would exceed the array is
refused before any work is queued.  This file is collected last so that a run
stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
import scan_gated_rnns_b200 as sgr
from scan_gated_rnns_b200 import _abi
from scan_gated_rnns_b200.synth import Workload, generate

from parity import TOL, rel_err

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = torch.device("cuda:0")


def call_noalloc(k, hx, h0, out):
    B, T, D = k.shape
    stream = torch.cuda.current_stream(k.device).cuda_stream
    return _abi.lib().mingru_scan_noalloc(k.data_ptr(), hx.data_ptr(), h0.data_ptr(), D,
                                          out.data_ptr(), B, T, D, _abi.SGR_F32, stream)


def unaligned(x):
    """The same values one element into a fresh buffer: rows no longer 16-byte aligned."""
    buf = torch.empty(x.numel() + 1, dtype=x.dtype, device=x.device)
    v = buf[1:].view(x.shape)
    v.copy_(x)
    return v


@pytest.mark.parametrize("shape,shift", [((8, 4096, 1024), False), ((3, 5000, 96), True)])
def test_noalloc_matches_the_oracle_on_two_calls(shape, shift):
    B, T, D = shape
    kernel = _abi.plan(_abi.SGR_OP_MINGRU, B, T, D, _abi.SGR_F32, not shift)["kernel"]
    assert kernel == (_abi.KERNEL_TILE if shift else _abi.KERNEL_PIPELINED)
    for seed in (101, 102):
        w = Workload("noalloc", "mingru", B, T, D, "f32", seed=seed, init="u01_1")
        k, hx, h0 = generate(w)
        kd, hd, h0d = k.to(DEV), hx.to(DEV), h0.to(DEV)
        if shift:
            kd, hd = unaligned(kd), unaligned(hd)
        out = torch.full((B, T, D), float("nan"), device=DEV)
        if shift:
            out = unaligned(out)
        assert call_noalloc(kd, hd, h0d, out) == _abi.SGR_OK
        torch.cuda.synchronize()
        ref = oracle.mingru_linear(k, hx, h0, threads=8)
        err = rel_err(out, ref)
        print(f"noalloc {shape} seed {seed}: max relative error {err:.3e}")
        assert err <= TOL["f32"]
        # and the workspace entry point on the same inputs agrees as closely
        same = sgr.mingru_scan(kd, hd, h0d)
        assert rel_err(out, same.double().cpu().numpy()) <= TOL["f32"]
        assert np.isfinite(out.cpu().numpy()).all()


def test_noalloc_refuses_shapes_beyond_its_scratch():
    # 4 x 2^22 rows of 512 channels needs far more than 16 MiB of hand-off words;
    # refused on the host before anything is queued (no memory is touched)
    B, T, D = 4, 1 << 22, 512
    assert _abi.lib().sgr_workspace_size(_abi.SGR_OP_MINGRU, B, T, D, _abi.SGR_F32) > 16 << 20
    # null operands: the size check comes first, and should it ever not, the
    # null check refuses the call before any launch
    code = _abi.lib().mingru_scan_noalloc(None, None, None, 0, None, B, T, D, _abi.SGR_F32, None)
    assert code == _abi.SGR_ERR_WORKSPACE
