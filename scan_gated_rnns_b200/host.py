"""Scans of tensors held in host memory (C ABI: mingru_scan_host,
minmax_scan_host): argument marshalling only.

    h = mingru_scan_host(k, hx, h0=None)      # k, hx: (B, T, D) CPU tensors
    x = minmax_scan_host(r, s, x0=None)

The library cuts the time axis into slices and overlaps each slice's upload,
scan and download on three CUDA streams (one of them PyTorch's current
stream); the device staging buffer it needs comes from PyTorch's allocator.
Page-locked inputs (``tensor.pin_memory()``) give overlapped copies; the
output is allocated page-locked when the inputs are.  With ``blocking=False``
the call returns once the work is enqueued and the output is complete when
the current stream reaches that point; the inputs must stay alive until then.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _abi
from ._abi import check, lib
from .ops import _DT, _dtype_code

_staging = {}


def staging_size(op: str, B: int, T: int, D: int, dtype: torch.dtype, chunks: int = 0) -> int:
    opc = {"mingru": _abi.SGR_OP_MINGRU, "minmax": _abi.SGR_OP_MINMAX}[op]
    return int(lib().sgr_host_staging_size(opc, B, T, D, _DT[dtype], chunks))


def _staging_buffer(device: torch.device, nbytes: int) -> torch.Tensor:
    """Device staging per (device, stream), grown on demand."""
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    buf = _staging.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        _staging[key] = buf
    return buf


def _host_rows(t: Optional[torch.Tensor], B: int, D: int, like: torch.Tensor, name: str):
    if t is None:
        return 0, 0
    if t.is_cuda or t.dtype != like.dtype:
        raise ValueError(f"{name} must be a CPU tensor of dtype {like.dtype}")
    if t.dim() == 1:
        if t.shape[0] != D or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous (D,) vector")
        return t.data_ptr(), 0
    if t.dim() != 2 or tuple(t.shape) != (B, D) or (D > 1 and t.stride(1) != 1):
        raise ValueError(f"{name} must be (B, D) = ({B}, {D}) with contiguous rows")
    return t.data_ptr(), (t.stride(0) if B > 1 else D)


def _scan_host(fn: str, op: str, p, q, init, out, chunks, device, blocking):
    for t, n in ((p, "first operand"), (q, "second operand")):
        if t.is_cuda or t.dim() != 3 or not t.is_contiguous():
            raise ValueError(f"{fn}: {n} must be a contiguous (B, T, D) CPU tensor")
    if p.shape != q.shape or p.dtype != q.dtype:
        raise ValueError(f"{fn}: operands must share shape and dtype")
    dt = _dtype_code(p, fn)
    B, T, D = p.shape
    ip, ibs = _host_rows(init, B, D, p, fn + ": initial state")
    if out is None:
        out = torch.empty(p.shape, dtype=p.dtype, pin_memory=p.is_pinned())
    elif out.is_cuda or out.shape != p.shape or out.dtype != p.dtype or not out.is_contiguous():
        raise ValueError(f"{fn}: out must be a contiguous CPU tensor like the operands")
    if p.numel() == 0:
        return out
    device = torch.device(device if device is not None else "cuda")
    if device.type != "cuda":
        raise ValueError(f"{fn}: device must be a CUDA device (the scans run on the GPU)")
    if device.index is None:
        device = torch.device("cuda", torch.cuda.current_device())
    need = staging_size(op, B, T, D, p.dtype, chunks)
    with torch.cuda.device(device):
        st = _staging_buffer(device, need)
        stream = torch.cuda.current_stream(device)
        code = getattr(lib(), fn)(p.data_ptr(), q.data_ptr(), ip, ibs, out.data_ptr(), B, T, D, dt,
                                  chunks, st.data_ptr(), st.numel(), stream.cuda_stream)
        check(fn, code)
        if blocking:
            stream.synchronize()
    return out


def mingru_scan_host(k: torch.Tensor, hx: torch.Tensor, h0: Optional[torch.Tensor] = None,
                     out: Optional[torch.Tensor] = None, chunks: int = 0, device=None,
                     blocking: bool = True) -> torch.Tensor:
    """minGRU scan of host (B, T, D) tensors, computed on the GPU; returns a
    host tensor.  ``chunks`` = time slices (0: automatic, about sqrt(input MiB / 4.6))."""
    return _scan_host("mingru_scan_host", "mingru", k, hx, h0, out, chunks, device, blocking)


def minmax_scan_host(r: torch.Tensor, s: torch.Tensor, x0: Optional[torch.Tensor] = None,
                     out: Optional[torch.Tensor] = None, chunks: int = 0, device=None,
                     blocking: bool = True) -> torch.Tensor:
    """MinMax scan of host (B, T, D) tensors (see mingru_scan_host)."""
    return _scan_host("minmax_scan_host", "minmax", r, s, x0, out, chunks, device, blocking)
