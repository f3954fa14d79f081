"""CPU oracle for the element-wise recurrence scans (minGRU, MinMax neuron).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product path under ``scan_gated_rnns_b200/`` never imports it, and the two
share no code.

The arithmetic lives in ``oracle.c`` (plain C, IEEE binary64, compiled with
``-ffp-contract=off`` so every product and sum is rounded on its own).  This
module only builds that file with gcc, loads it with ctypes and marshals numpy
arrays in and out.

Functions (all inputs are widened exactly to float64 first):

``mingru_linear(k, hx, h0=None)``
    minGRU recurrence h_t = (1 - z_t) h_{t-1} + z_t g(hx_t), z_t = sigmoid(k_t),
    g(x) = x + 0.5 (x >= 0) or sigmoid(x) (x < 0); page "Mingru Pytorch"
    (Requirements & limits; Install and apply the minGRU layer).
``mingru_log(k, hx, h0=None)``
    the same quantity through the log-space formula
    h_t = exp(a*_t + logcumsumexp(log z + log g(hx) - a*)), a* = cumsum(-softplus(k)).
``minmax(r, s, x0=None)``
    MinMax neuron x_{t+1} = max(min(r_t, x_t), s_t); page "MinMax Recurrent
    Neural Cascades" (The model, item 3).
``mingru_decay(k, hx, h0, dt, lam, log1p_delta=False)``
    minGRU with time decay: the state is gated by gamma_t = exp(-lam_d u_bt)
    (u = dt or log1p(dt); lam u > 1e4 wipes it) at each token boundary; page
    "Your first delta model", Step 5.  ``mingru_decay_backward`` adds dlam.
``mingru_projected(x, w, h0=None)``
    the minGRU layer's input projection and scan: k = x W[:D]^T, hx = x W[D:]^T
    (fp64 matrix products, numpy), then ``mingru_linear``; page "Mingru
    Pytorch" (the layer applied to a (B, T, d) input).
``mingru_backward(k, hx, h0, gy)`` / ``minmax_backward(r, s, x0, gy)``
    gradients of a loss with dL/d out = gy with respect to both inputs and the
    initial state, by the chain rule through the sequential loop (forward
    recomputed in fp64); MinMax ties share the gradient evenly, as PyTorch's
    elementwise minimum/maximum do.

Arrays are (B, T, D); optional states are (B, D).  ``threads`` splits the batch
over Python threads (ctypes releases the GIL during the C call).
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc); return the path."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _open(path: str):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.c_int64
    for name in ("oracle_mingru_linear", "oracle_mingru_log", "oracle_minmax"):
        fn = getattr(lib, name)
        fn.restype = ctypes.c_int
        fn.argtypes = [dp, dp, dp, i64, dp, i64, i64, i64]
    for name in ("oracle_mingru_backward", "oracle_minmax_backward"):
        fn = getattr(lib, name)
        fn.restype = ctypes.c_int
        fn.argtypes = [dp, dp, dp, i64, dp, dp, dp, dp, i64, i64, i64]
    lib.oracle_mingru_decay.restype = ctypes.c_int
    lib.oracle_mingru_decay.argtypes = [dp, dp, dp, i64, dp, i64, dp, ctypes.c_int, dp, i64, i64, i64]
    lib.oracle_mingru_decay_backward.restype = ctypes.c_int
    lib.oracle_mingru_decay_backward.argtypes = [dp, dp, dp, i64, dp, i64, dp, ctypes.c_int, dp, dp, dp,
                                                 dp, dp, i64, i64, i64]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _open(build())
    return _lib


@contextlib.contextmanager
def use_library(path: str):
    """Run the oracle functions against another build of oracle.c (the pin
    suite uses this to show that planted mistakes are caught)."""
    global _lib
    _load()
    with _lock:
        saved, _lib = _lib, _open(path)
    try:
        yield
    finally:
        with _lock:
            _lib = saved


def _as_f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor: widen on the torch side (exact for bf16/fp32)
        import torch
        a = a.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _run(name: str, p, q, init, threads: int) -> np.ndarray:
    p = _as_f64(p)
    q = _as_f64(q)
    if p.ndim != 3 or p.shape != q.shape:
        raise ValueError(f"inputs must be two (B, T, D) arrays of one shape, got {p.shape} {q.shape}")
    B, T, D = p.shape
    out = np.empty_like(p)
    if init is not None:
        init = _as_f64(init).reshape(B, D)
    fn = getattr(_load(), name)

    def one(b0: int, b1: int) -> None:
        nb = b1 - b0
        if nb <= 0:
            return
        ip = _ptr(init[b0:b1]) if init is not None else None
        rc = fn(_ptr(p[b0:b1]), _ptr(q[b0:b1]), ip, D, _ptr(out[b0:b1]), nb, T, D)
        if rc != 0:
            raise RuntimeError(f"{name} returned {rc}")

    threads = max(1, min(int(threads), B)) if B > 0 else 1
    if threads == 1:
        one(0, B)
    else:
        bounds = np.linspace(0, B, threads + 1).astype(int)
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda i: one(bounds[i], bounds[i + 1]), range(threads)))
    return out


def mingru_linear(k, hx, h0=None, threads: int = 1) -> np.ndarray:
    """fp64 sequential minGRU recurrence (linear space)."""
    return _run("oracle_mingru_linear", k, hx, h0, threads)


def mingru_log(k, hx, h0=None, threads: int = 1) -> np.ndarray:
    """fp64 minGRU through the log-space formula (finite k; h0 > 0 if given)."""
    return _run("oracle_mingru_log", k, hx, h0, threads)


def minmax(r, s, x0=None, threads: int = 1) -> np.ndarray:
    """MinMax neuron scan, out[t] = x_{t+1} (exact: selection only)."""
    return _run("oracle_minmax", r, s, x0, threads)


def mingru_step(k_t, hx_t, h_prev=None) -> np.ndarray:
    """One token of the recurrence: the linear oracle on a length-1 sequence."""
    k_t = _as_f64(k_t)
    hx_t = _as_f64(hx_t)
    B, D = k_t.shape
    h = mingru_linear(k_t.reshape(B, 1, D), hx_t.reshape(B, 1, D), h_prev)
    return h.reshape(B, D)


def _run_backward(name: str, p, q, init, gy, threads: int):
    p, q, gy = _as_f64(p), _as_f64(q), _as_f64(gy)
    if p.ndim != 3 or p.shape != q.shape or p.shape != gy.shape:
        raise ValueError(f"inputs must be three (B, T, D) arrays of one shape, got {p.shape} {q.shape} {gy.shape}")
    B, T, D = p.shape
    dp, dq = np.empty_like(p), np.empty_like(p)
    dinit = np.empty((B, D), dtype=np.float64)
    if init is not None:
        init = _as_f64(init).reshape(B, D)
    fn = getattr(_load(), name)

    def one(b0: int, b1: int) -> None:
        if b1 <= b0:
            return
        ip = _ptr(init[b0:b1]) if init is not None else None
        rc = fn(_ptr(p[b0:b1]), _ptr(q[b0:b1]), ip, D, _ptr(gy[b0:b1]), _ptr(dp[b0:b1]),
                _ptr(dq[b0:b1]), _ptr(dinit[b0:b1]), b1 - b0, T, D)
        if rc != 0:
            raise RuntimeError(f"{name} returned {rc}")

    threads = max(1, min(int(threads), B)) if B > 0 else 1
    if threads == 1:
        one(0, B)
    else:
        bounds = np.linspace(0, B, threads + 1).astype(int)
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda i: one(bounds[i], bounds[i + 1]), range(threads)))
    return dp, dq, dinit


def mingru_backward(k, hx, h0, gy, threads: int = 1):
    """(dk, dhx, dh0) of a loss with dL/dh = gy (fp64; dh0 is (B, D) whether
    or not h0 is given: the gradient with respect to the initial state)."""
    return _run_backward("oracle_mingru_backward", k, hx, h0, gy, threads)


def minmax_backward(r, s, x0, gy, threads: int = 1):
    """(dr, ds, dx0) of a loss with dL/d out = gy (fp64; ties share evenly)."""
    return _run_backward("oracle_minmax_backward", r, s, x0, gy, threads)


def _decay_args(dt, lam, B, T, D):
    dt = _as_f64(dt).reshape(B, T)
    lam = _as_f64(lam).reshape(D)
    return dt, lam


def mingru_decay(k, hx, h0, dt, lam, log1p_delta: bool = False) -> np.ndarray:
    """fp64 minGRU with time decay; dt (B, T) gaps, lam (D,) rates."""
    k, hx = _as_f64(k), _as_f64(hx)
    B, T, D = k.shape
    dt, lam = _decay_args(dt, lam, B, T, D)
    init = _as_f64(h0).reshape(B, D) if h0 is not None else None
    h = np.empty_like(k)
    rc = _load().oracle_mingru_decay(_ptr(k), _ptr(hx), _ptr(init) if init is not None else None, D,
                                     _ptr(dt), T, _ptr(lam), int(log1p_delta), _ptr(h), B, T, D)
    if rc != 0:
        raise RuntimeError(f"oracle_mingru_decay returned {rc}")
    return h


def mingru_decay_backward(k, hx, h0, dt, lam, gy, log1p_delta: bool = False):
    """(dk, dhx, dh0, dlam) of a loss with dL/dh = gy through mingru_decay."""
    k, hx, gy = _as_f64(k), _as_f64(hx), _as_f64(gy)
    B, T, D = k.shape
    dt, lam = _decay_args(dt, lam, B, T, D)
    init = _as_f64(h0).reshape(B, D) if h0 is not None else None
    dk, dhx = np.empty_like(k), np.empty_like(k)
    dh0, dlam = np.empty((B, D)), np.empty(D)
    rc = _load().oracle_mingru_decay_backward(
        _ptr(k), _ptr(hx), _ptr(init) if init is not None else None, D, _ptr(dt), T, _ptr(lam),
        int(log1p_delta), _ptr(gy), _ptr(dk), _ptr(dhx), _ptr(dh0), _ptr(dlam), B, T, D)
    if rc != 0:
        raise RuntimeError(f"oracle_mingru_decay_backward returned {rc}")
    return dk, dhx, dh0, dlam


def mingru_projected(x, w, h0=None, threads: int = 1) -> np.ndarray:
    """fp64: the projections k = x w[:D]^T and hx = x w[D:]^T of a (B, T, d_in)
    input by a (2 D, d_in) weight, then the minGRU recurrence."""
    x, w = _as_f64(x), _as_f64(w)
    if x.ndim != 3 or w.ndim != 2 or w.shape[1] != x.shape[2] or w.shape[0] % 2:
        raise ValueError(f"x must be (B, T, d_in) and w (2 D, d_in), got {x.shape} {w.shape}")
    D = w.shape[0] // 2
    k = np.ascontiguousarray(x @ w[:D].T)
    hx = np.ascontiguousarray(x @ w[D:].T)
    return mingru_linear(k, hx, h0, threads=threads)
