"""Differentiable wrappers: torch.autograd.Function around the forward scans
and their gradient kernels (argument marshalling only; both directions run
in libsgr.so).

    h = mingru_scan_fn(k, hx, h0)      # h.backward() reaches k, hx and h0
    x = minmax_scan_fn(r, s, x0)

The forward output is kept for the backward pass (the gradient kernels read
the state before each step from it), so a differentiable call holds one
extra (B, T, D) tensor until backward.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import ops


def _init_grad(dinit: torch.Tensor, init: Optional[torch.Tensor]):
    if init is None:
        return None
    if init.dim() == 1:      # one (D,) state broadcast to every batch row
        return dinit.sum(0)
    return dinit


class MinGRUScan(torch.autograd.Function):
    @staticmethod
    def forward(ctx, k, hx, h0=None):
        h = ops.mingru_scan(k, hx, h0)
        ctx.save_for_backward(k, hx, h0, h)
        return h

    @staticmethod
    def backward(ctx, dh):
        k, hx, h0, h = ctx.saved_tensors
        dk, dhx, dh0 = ops.mingru_scan_backward(k, hx, h0, h, dh.contiguous(),
                                                want_dh0=h0 is not None and ctx.needs_input_grad[2])
        return dk, dhx, (_init_grad(dh0, h0) if dh0 is not None else None)


class MinMaxScan(torch.autograd.Function):
    @staticmethod
    def forward(ctx, r, s, x0=None):
        x = ops.minmax_scan(r, s, x0)
        ctx.save_for_backward(r, s, x0, x)
        return x

    @staticmethod
    def backward(ctx, dx):
        r, s, x0, x = ctx.saved_tensors
        dr, ds, dx0 = ops.minmax_scan_backward(r, s, x0, x, dx.contiguous(),
                                               want_dx0=x0 is not None and ctx.needs_input_grad[2])
        return dr, ds, (_init_grad(dx0, x0) if dx0 is not None else None)


class MinGRUDecayScan(torch.autograd.Function):
    @staticmethod
    def forward(ctx, k, hx, h0, delta_t, lam, log1p_delta):
        h = ops.mingru_scan_decay(k, hx, h0, delta_t, lam, log1p_delta)
        ctx.save_for_backward(k, hx, h0, delta_t, lam, h)
        ctx.log1p_delta = log1p_delta
        return h

    @staticmethod
    def backward(ctx, dh):
        k, hx, h0, delta_t, lam, h = ctx.saved_tensors
        dk, dhx, dh0, dlam = ops.mingru_scan_decay_backward(
            k, hx, h0, delta_t, lam, h, dh.contiguous(), ctx.log1p_delta,
            want_dh0=h0 is not None and ctx.needs_input_grad[2], want_dlam=ctx.needs_input_grad[4])
        return (dk, dhx, (_init_grad(dh0, h0) if dh0 is not None else None), None, dlam, None)


def mingru_scan_decay_fn(k: torch.Tensor, hx: torch.Tensor, h0: Optional[torch.Tensor],
                         delta_t: torch.Tensor, lam: torch.Tensor,
                         log1p_delta: bool = False) -> torch.Tensor:
    """mingru_scan_decay with gradients for k, hx, h0 and lam (not delta_t)."""
    return MinGRUDecayScan.apply(k, hx, h0, delta_t, lam, log1p_delta)


def mingru_scan_fn(k: torch.Tensor, hx: torch.Tensor, h0: Optional[torch.Tensor] = None) -> torch.Tensor:
    """mingru_scan with gradients for k, hx and h0."""
    return MinGRUScan.apply(k, hx, h0)


def minmax_scan_fn(r: torch.Tensor, s: torch.Tensor, x0: Optional[torch.Tensor] = None) -> torch.Tensor:
    """minmax_scan with gradients for r, s and x0."""
    return MinMaxScan.apply(r, s, x0)
