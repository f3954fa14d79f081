"""mingru_scan_noalloc: the scan for callers that cannot allocate device memory
where they run it (a runtime plugin whose enqueue step must not allocate, a
fixed device-memory plan, code running under stream capture).  Its scratch is
a fixed array inside the library instead of a caller-provided workspace.

Checked through the C ABI against mingru_scan on the same inputs, on two calls
in a row (the second reuses the array the first left behind), within the fp32
parity tolerance of the other tests; and a shape whose scratch would exceed
the array is refused before any work is queued.  This file is collected last
so that a run stopping at the first failure has already run every other test.
"""
import pytest
import torch

import scan_gated_rnns_b200 as sgr
from scan_gated_rnns_b200 import _abi
from scan_gated_rnns_b200.synth import Workload, generate

from parity import TOL, rel_err

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def call_noalloc(k, hx, h0, out):
    B, T, D = k.shape
    stream = torch.cuda.current_stream(k.device).cuda_stream
    return _abi.lib().mingru_scan_noalloc(k.data_ptr(), hx.data_ptr(), h0.data_ptr(), D,
                                          out.data_ptr(), B, T, D, _abi.SGR_F32, stream)


def test_noalloc_matches_mingru_scan_on_two_calls():
    dev = torch.device("cuda:0")
    for seed in (101, 102):
        w = Workload("noalloc", "mingru", 8, 4096, 1024, "f32", seed=seed, init="u01_1")
        k, hx, h0 = generate(w, device=dev)
        ref = sgr.mingru_scan(k, hx, h0)
        out = torch.full_like(k, float("nan"))
        assert call_noalloc(k, hx, h0, out) == _abi.SGR_OK
        torch.cuda.synchronize()
        assert rel_err(out, ref.double().cpu().numpy()) <= TOL["f32"]


def test_noalloc_refuses_shapes_beyond_its_scratch():
    # 4 x 2^22 rows of 512 channels needs far more than 16 MiB of hand-off words;
    # refused on the host before anything is queued (no memory is touched)
    B, T, D = 4, 1 << 22, 512
    assert _abi.lib().sgr_workspace_size(_abi.SGR_OP_MINGRU, B, T, D, _abi.SGR_F32) > 16 << 20
    code = _abi.lib().mingru_scan_noalloc(0x10000000, 0x20000000, None, 0, 0x30000000,
                                          B, T, D, _abi.SGR_F32, None)
    assert code == _abi.SGR_ERR_WORKSPACE
