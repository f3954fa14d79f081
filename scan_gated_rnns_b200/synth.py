"""Seeded synthetic inputs for the scans.

This module is shared by the tests, the benchmark and the smoke check, and
feeds both the CUDA library and the CPU oracle.  It holds none of the scans'
arithmetic: it only draws random numbers with a seeded ``torch.Generator``
and rounds them to the I/O dtype.

Draw order per workload: first operand (k or r), second operand (hx or s),
then the optional initial state.  bf16 inputs are fp32 draws rounded to
nearest-even by ``Tensor.to``; the identical bits go to the GPU and the oracle.
Draws are made on the device asked for (a CPU or a CUDA ``torch.Generator``
seeded the same way); the two devices give different numbers for one seed,
so a run that checks GPU results copies the GPU-drawn inputs to the host for
the oracle rather than drawing them twice.

The named workloads are the shapes and distributions of the minGRU layer
example on the page "Mingru Pytorch" (batched (B, T, D) tensors such as
torch.randn(2, 1024, 512)) and of the MinMax neuron on the page "MinMax
Recurrent Neural Cascades" (d_model 768 in its custom configuration), widened
to the sizes the benchmark and the parity tests use.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional

import torch

_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    op: str            # "mingru" or "minmax"
    B: int
    T: int
    D: int
    dtype: str         # "f32" or "bf16" (I/O dtype; arithmetic is fp32 on the GPU)
    seed: int
    k_mean: float = 0.0     # mean of k (minGRU) -- N(k_mean, 1)
    init: Optional[str] = None  # None: no initial state; "u01_1": U(0.1, 1.0); "zero": explicit zeros

    @property
    def n_elems(self) -> int:
        return self.B * self.T * self.D

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def algorithmic_bytes(self) -> int:
        """Bytes a scan must move once each: two inputs read, one output written,
        plus the (B, D) initial state if one is passed."""
        b = 3 * self.n_elems * self.elem_bytes
        if self.init is not None:
            b += self.B * self.D * self.elem_bytes
        return b

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("mingru_b2_t1024_d512_f32", "mingru", 2, 1024, 512, "f32", seed=0),
        Workload("mingru_b8_t4096_d1024_f32_h0", "mingru", 8, 4096, 1024, "f32", seed=1, init="u01_1"),
        Workload("minmax_b4_t8192_d768_f32", "minmax", 4, 8192, 768, "f32", seed=2),
        Workload("mingru_b1_t131072_d512_f32_h0", "mingru", 1, 131072, 512, "f32", seed=3,
                 k_mean=2.0, init="u01_1"),
        Workload("mingru_b16_t2048_d4096_bf16_h0", "mingru", 16, 2048, 4096, "bf16", seed=4,
                 init="u01_1"),
    ]
}

# the workload the benchmark times by default: the largest single-GPU shape,
# the minGRU scan of B16 x T2048 x D4096 with bf16 I/O and a carried state
BENCH_WORKLOAD = "mingru_b16_t2048_d4096_bf16_h0"


def generate(w: Workload, seed: Optional[int] = None, device="cpu"):
    """Return (p, q, init) tensors on `device` in the workload's I/O dtype.

    p, q are (B, T, D): (k, hx) for minGRU with k ~ N(k_mean, 1), hx ~ N(0, 1);
    (r, s) for MinMax with r, s ~ N(0, 1).  init is (B, D) or None.
    """
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    shape = (w.B, w.T, w.D)
    p = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    if w.k_mean:
        p += w.k_mean
    q = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    init = None
    if w.init == "u01_1":
        init = torch.rand((w.B, w.D), generator=g, dtype=torch.float32, device=device) * 0.9 + 0.1
    elif w.init == "zero":
        init = torch.zeros((w.B, w.D), dtype=torch.float32, device=device)
    dt = _DTYPES[w.dtype]
    p, q = p.to(dt), q.to(dt)
    if init is not None:
        init = init.to(dt)
    return p, q, init


def sample_channels(w: Workload, n: int, seed: int = 1234):
    """n distinct (b, d) channel indices, seeded; always includes the first and
    the last channel so both ends of the D range are covered."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    total = w.B * w.D
    n = min(n, total)
    idx = torch.randperm(total, generator=g)[:n].tolist()
    idx = sorted(set(idx) | {0, total - 1})
    return [(i // w.D, i % w.D) for i in idx]
