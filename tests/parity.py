"""Shared helpers of the GPU parity tests: tolerances, error measures and the
oracle evaluated on a sample of channels."""
import numpy as np
import torch

import oracle

# minGRU parity bars: max relative error vs the fp64 oracle
TOL = {"f32": 1e-5, "bf16": 2e-2}
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def rel_err(got, ref) -> float:
    """max |got - ref| / max(|ref|, 1e-30) over all elements (fp64)."""
    if hasattr(got, "detach"):
        got = got.detach().to("cpu", torch.float64).numpy()
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if got.size == 0:
        return 0.0
    if not np.isfinite(got).all():
        return float("inf")
    return float(np.max(np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)))


def channels(x: torch.Tensor, chans):
    """(n, T, 1) fp64 host array of the listed (b, d) channels of a (B, T, D)
    tensor (input values are copied, never recomputed)."""
    b = torch.tensor([c[0] for c in chans], device=x.device)
    d = torch.tensor([c[1] for c in chans], device=x.device)
    return x[b, :, d].to("cpu", torch.float64).numpy()[:, :, None]


def init_rows(init: torch.Tensor, chans):
    if init is None:
        return None
    b = torch.tensor([c[0] for c in chans], device=init.device)
    d = torch.tensor([c[1] for c in chans], device=init.device)
    return init[b, d].to("cpu", torch.float64).numpy()[:, None]


def oracle_on_channels(op, p, q, init, chans, threads=8):
    """Oracle over the full T of a sample of channels: (n, T) fp64."""
    P, Q, I = channels(p, chans), channels(q, chans), init_rows(init, chans)
    if op == "mingru":
        out = oracle.mingru_linear(P, Q, I, threads=threads)
    else:
        out = oracle.minmax(P, Q, I, threads=threads)
    return out[:, :, 0]


def gpu_channels(y: torch.Tensor, chans):
    b = torch.tensor([c[0] for c in chans], device=y.device)
    d = torch.tensor([c[1] for c in chans], device=y.device)
    return y[b, :, d].to("cpu", torch.float64).numpy()


def _as_host(x):
    if hasattr(x, "detach"):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _fold_channels(a, G):
    """(B, T, D) -> (B G, T, D / G): channel groups become batch rows, so the
    oracle's threads (one per batch row) all have work."""
    B, T, D = a.shape
    return a.reshape(B, T, G, D // G).transpose(0, 2, 1, 3).reshape(B * G, T, D // G)


def _unfold_channels(a, B, G):
    BG, T, Dg = a.shape
    return a.reshape(B, G, T, Dg).transpose(0, 2, 1, 3).reshape(B, T, G * Dg)


def full_rel_err(op, p, q, init, got, threads=8, rows=2, fn=None):
    """Max relative error of `got` (B, T, D) against the oracle over EVERY
    channel and row, evaluated `rows` batch rows at a time (bounded host
    memory).  `fn` replaces the oracle call (same signature as
    oracle.mingru_linear) for other recurrences."""
    B, T, D = p.shape
    call = fn or (oracle.mingru_linear if op == "mingru" else oracle.minmax)
    worst = 0.0
    for b0 in range(0, B, rows):
        b1 = min(B, b0 + rows)
        nb = b1 - b0
        G = 1
        while nb * G < threads and D % (2 * G) == 0 and D // (2 * G) >= 8:
            G *= 2
        P = _fold_channels(_as_host(p[b0:b1]), G)
        Q = _fold_channels(_as_host(q[b0:b1]), G)
        I = None
        if init is not None:
            I = _as_host(init[b0:b1]).reshape(nb * G, D // G)
        ref = _unfold_channels(call(P, Q, I, threads=threads), nb, G)
        worst = max(worst, rel_err(got[b0:b1], ref))
    return worst
