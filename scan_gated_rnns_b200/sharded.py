"""Scans of sequences whose time axis is split across ranks (one GPU each):
argument marshalling and the exchange; the arithmetic runs in libsgr.so.

    h_local = time_sharded_scan("mingru", k_local, hx_local, h0, group)

Rank r holds steps [t_r, t_{r+1}) of every channel (contiguous slices in rank
order; slices may differ in length).  Each rank (1) summarises its slice per
channel into one pair (sgr_scan_summary: minGRU h_end = A h_start + B, MinMax
x_end = max(min(x_start, U), L)), (2) all-gathers the (B, D, 2) pairs over
the process group (NCCL for CUDA tensors), (3) applies the pairs of the ranks
before it to the initial state (sgr_combine_summaries), and (4) scans its
slice from that state.  Step 1 reads the slice once more than a single-device
scan; the exchange moves 8 B D bytes per rank.

`ops` replaces the three device steps (summary, combine, scan); the default is
this package's CUDA library.  Tests of the exchange on CPU ranks pass their
own.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import _abi, ops as _ops
from ._abi import check, lib

_OP = {"mingru": _abi.SGR_OP_MINGRU, "minmax": _abi.SGR_OP_MINMAX}


def scan_summary(op: str, p: torch.Tensor, q: torch.Tensor) -> torch.Tensor:
    """(B, D, 2) float32 pairs summarising the (B, T, D) slice p, q."""
    _ops._seq(p, "scan_summary: first operand")
    _ops._seq(q, "scan_summary: second operand")
    if p.shape != q.shape or p.dtype != q.dtype or p.device != q.device:
        raise ValueError("scan_summary: operands must share shape, dtype and device")
    dt = _ops._dtype_code(p, "scan_summary")
    B, T, D = p.shape
    pairs = torch.empty((B, D, 2), dtype=torch.float32, device=p.device)
    need = int(lib().sgr_summary_workspace_size(B, max(T, 1), D, dt))
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=p.device)
    with torch.cuda.device(p.device):
        code = lib().sgr_scan_summary(_OP[op], p.data_ptr(), q.data_ptr(), B, T, D, dt,
                                      pairs.data_ptr(), ws.data_ptr(), ws.numel(),
                                      _ops._stream(p.device))
    check("sgr_scan_summary", code)
    return pairs


def combine_summaries(op: str, pairs: torch.Tensor, rank: int, init: Optional[torch.Tensor],
                      dtype: torch.dtype) -> torch.Tensor:
    """(B, D) state entering slice `rank` from all slices' pairs (n, B, D, 2)."""
    if pairs.dim() != 4 or pairs.shape[-1] != 2 or pairs.dtype != torch.float32 or not pairs.is_contiguous():
        raise ValueError("combine_summaries: pairs must be a contiguous (n, B, D, 2) float32 tensor")
    _ops._need_cuda(pairs, "combine_summaries: pairs")
    n, B, D, _ = pairs.shape
    if not 0 <= rank < n:
        raise ValueError(f"combine_summaries: rank {rank} outside 0..{n - 1}")
    like = torch.empty(0, dtype=dtype, device=pairs.device)
    ip, ibs = _ops._rows(init, B, D, like, "combine_summaries: initial state")
    out = torch.empty((B, D), dtype=dtype, device=pairs.device)
    dt = _ops._DT[dtype]
    with torch.cuda.device(pairs.device):
        code = lib().sgr_combine_summaries(_OP[op], pairs.data_ptr(), rank, ip, ibs, out.data_ptr(),
                                           D, B, D, dt, _ops._stream(pairs.device))
    check("sgr_combine_summaries", code)
    return out


class DeviceOps:
    """The three per-rank steps, on this package's CUDA library."""

    @staticmethod
    def summary(op, p, q):
        return scan_summary(op, p, q)

    @staticmethod
    def combine(op, pairs, rank, init, dtype):
        return combine_summaries(op, pairs, rank, init, dtype)

    @staticmethod
    def scan(op, p, q, init):
        return (_ops.mingru_scan if op == "mingru" else _ops.minmax_scan)(p, q, init)


def time_sharded_scan(op: str, p_local: torch.Tensor, q_local: torch.Tensor,
                      init: Optional[torch.Tensor] = None, group=None, ops=DeviceOps) -> torch.Tensor:
    """Outputs of this rank's slice of a scan whose time axis is split over the
    ranks of `group` in rank order.  `init` is the sequence's initial state
    (the same on every rank; only the first slice starts from it)."""
    if op not in _OP:
        raise ValueError(f"unknown op {op!r}")
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    pairs = ops.summary(op, p_local, q_local).contiguous()
    gathered = [torch.empty_like(pairs) for _ in range(world)]
    dist.all_gather(gathered, pairs, group=group)
    h_in = ops.combine(op, torch.stack(gathered, 0).contiguous(), rank, init, p_local.dtype)
    return ops.scan(op, p_local, q_local, h_in)
