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
