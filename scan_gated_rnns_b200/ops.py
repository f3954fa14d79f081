"""Torch-facing wrappers of the C ABI: argument marshalling only.

Every operation runs in the CUDA library (``libsgr.so``).  These wrappers check
shapes, dtypes and devices, allocate outputs and the workspace with PyTorch's
allocator, pass raw device pointers and PyTorch's current stream, and turn a
non-zero status into an exception.  There is no CPU path.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import _abi
from ._abi import check, lib

_DT = {torch.float32: _abi.SGR_F32, torch.bfloat16: _abi.SGR_BF16}


def _dtype_code(t: torch.Tensor, name: str) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"{name}: dtype {t.dtype} is not supported (float32 or bfloat16)") from None


def _need_cuda(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the scans have no CPU path)")


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _seq(t: torch.Tensor, name: str) -> None:
    _need_cuda(t, name)
    if t.dim() != 3:
        raise ValueError(f"{name} must be (B, T, D), got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (B, T, D)")


def _rows(t: Optional[torch.Tensor], B: int, D: int, like: torch.Tensor, name: str) -> Tuple[int, int]:
    """(pointer, batch stride in elements) of a (B, D) or (D,) operand.  (On
    the decode step's path: one stride tuple and integer device indices keep
    it to a few attribute reads.)"""
    if t is None:
        return 0, 0
    _need_cuda(t, name)
    if t.dtype != like.dtype or t.get_device() != like.get_device():
        raise ValueError(f"{name} must have dtype {like.dtype} on {like.device}")
    st = t.stride()
    if len(st) == 1:
        if t.shape[0] != D or (D > 1 and st[0] != 1):
            raise ValueError(f"{name} must be a contiguous (D,) vector")
        return t.data_ptr(), 0
    if len(st) != 2 or t.shape != (B, D):
        raise ValueError(f"{name} must be (B, D) = ({B}, {D}), got {tuple(t.shape)}")
    if D > 1 and st[1] != 1:
        raise ValueError(f"{name} rows must be contiguous along D")
    return t.data_ptr(), (st[0] if B > 1 else D)


class Workspace:
    """Device workspace of the chunked scans, zero-filled when allocated (the
    library keeps it valid from call to call).  Use one per stream."""

    def __init__(self, nbytes: int, device) -> None:
        self.nbytes = max(int(nbytes), 256)
        self.buf = torch.zeros(self.nbytes, dtype=torch.uint8, device=device)

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()

    def status(self, clear: bool = True) -> int:
        """Synchronise the current stream and return the device status word
        (0 = ok, SGR_ERR_TIMEOUT if a chunk gave up waiting)."""
        return lib().sgr_workspace_status(self.ptr, self.nbytes, int(clear), _stream(self.buf.device))


_cache = {}


def workspace_size(op: str, B: int, T: int, D: int, dtype: torch.dtype) -> int:
    opc = {"mingru": _abi.SGR_OP_MINGRU, "minmax": _abi.SGR_OP_MINMAX, "mingru_log": _abi.SGR_OP_MINGRU_LOG}[op]
    return int(lib().sgr_workspace_size(opc, B, T, D, _DT[dtype]))


def default_workspace(device: torch.device, nbytes: int) -> Workspace:
    """The per-(device, stream) workspace the wrappers use when none is given."""
    key = (device.index, _stream(device))
    ws = _cache.get(key)
    if ws is None or ws.nbytes < nbytes:
        ws = Workspace(nbytes, device)
        _cache[key] = ws
    return ws


def _scan(fn: str, op: int, p: torch.Tensor, q: torch.Tensor, init, out, workspace):
    _seq(p, fn + ": first operand")
    _seq(q, fn + ": second operand")
    if p.shape != q.shape or p.dtype != q.dtype or p.device != q.device:
        raise ValueError(f"{fn}: operands must share shape, dtype and device")
    dt = _dtype_code(p, fn)
    B, T, D = p.shape
    ip, ibs = _rows(init, B, D, p, fn + ": initial state")
    if out is None:
        out = torch.empty_like(p)
    else:
        _seq(out, fn + ": out")
        if out.shape != p.shape or out.dtype != p.dtype or out.device != p.device:
            raise ValueError(f"{fn}: out must match the operands")
    need = int(lib().sgr_workspace_size(op, B, T, D, dt))
    wp, wn = 0, 0
    if need or workspace is not None:
        # a workspace given where none is needed still receives the status word
        ws = workspace if workspace is not None else default_workspace(p.device, need)
        wp, wn = ws.ptr, ws.nbytes
    with torch.cuda.device(p.device):
        code = getattr(lib(), fn)(p.data_ptr(), q.data_ptr(), ip, ibs, out.data_ptr(),
                                  B, T, D, dt, wp, wn, _stream(p.device))
    check(fn, code)
    return out


def mingru_scan(k: torch.Tensor, hx: torch.Tensor, h0: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, workspace: Optional[Workspace] = None) -> torch.Tensor:
    """h (B, T, D): minGRU over the time axis of pre-activations k, hx (B, T, D),
    with optional initial state h0 (B, D) or (D,)."""
    return _scan("mingru_scan", _abi.SGR_OP_MINGRU, k, hx, h0, out, workspace)


def mingru_scan_log(k: torch.Tensor, hx: torch.Tensor, h0: Optional[torch.Tensor] = None,
                    out: Optional[torch.Tensor] = None, workspace: Optional[Workspace] = None) -> torch.Tensor:
    """mingru_scan's result evaluated in log space (log2 h carried through the
    chunked kernels); h0 must be >= 0."""
    return _scan("mingru_scan_log", _abi.SGR_OP_MINGRU_LOG, k, hx, h0, out, workspace)


def minmax_scan(r: torch.Tensor, s: torch.Tensor, x0: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, workspace: Optional[Workspace] = None) -> torch.Tensor:
    """x (B, T, D), x[:, t] = x_{t+1} = max(min(r_t, x_t), s_t), x_0 = x0 or +0."""
    return _scan("minmax_scan", _abi.SGR_OP_MINMAX, r, s, x0, out, workspace)


def _scan_backward(fn: str, op: int, p, q, init, fwd, gy, want_dinit: bool, workspace):
    for t, n in ((p, "first operand"), (q, "second operand"), (fwd, "forward output"),
                 (gy, "upstream gradient")):
        _seq(t, f"{fn}: {n}")
        if t.shape != p.shape or t.dtype != p.dtype or t.device != p.device:
            raise ValueError(f"{fn}: {n} must match the first operand's shape, dtype and device")
    dt = _dtype_code(p, fn)
    B, T, D = p.shape
    ip, ibs = _rows(init, B, D, p, fn + ": initial state")
    dp, dq = torch.empty_like(p), torch.empty_like(p)
    dinit = torch.empty((B, D), dtype=p.dtype, device=p.device) if want_dinit else None
    need = int(lib().sgr_backward_workspace_size(op, B, T, D, dt))
    wp, wn = 0, 0
    if need:
        ws = workspace if workspace is not None else default_workspace(p.device, need)
        wp, wn = ws.ptr, ws.nbytes
    with torch.cuda.device(p.device):
        code = getattr(lib(), fn)(p.data_ptr(), q.data_ptr(), ip, ibs, fwd.data_ptr(), gy.data_ptr(),
                                  dp.data_ptr(), dq.data_ptr(),
                                  dinit.data_ptr() if dinit is not None else 0, D,
                                  B, T, D, dt, wp, wn, _stream(p.device))
    check(fn, code)
    return dp, dq, dinit


def mingru_scan_backward(k: torch.Tensor, hx: torch.Tensor, h0: Optional[torch.Tensor],
                         h: torch.Tensor, dh: torch.Tensor, want_dh0: bool = True,
                         workspace: Optional[Workspace] = None):
    """(dk, dhx, dh0) for dL/dh = dh through h = mingru_scan(k, hx, h0); dh0 is
    (B, D) (or None when want_dh0 is false)."""
    return _scan_backward("mingru_scan_backward", _abi.SGR_OP_MINGRU, k, hx, h0, h, dh, want_dh0,
                          workspace)


def minmax_scan_backward(r: torch.Tensor, s: torch.Tensor, x0: Optional[torch.Tensor],
                         x: torch.Tensor, dx: torch.Tensor, want_dx0: bool = True,
                         workspace: Optional[Workspace] = None):
    """(dr, ds, dx0) for dL/dx = dx through x = minmax_scan(r, s, x0); equal
    operands of a min or a max share the gradient evenly."""
    return _scan_backward("minmax_scan_backward", _abi.SGR_OP_MINMAX, r, s, x0, x, dx, want_dx0,
                          workspace)


def _decay_operands(fn: str, p: torch.Tensor, delta_t: torch.Tensor, lam: torch.Tensor):
    B, T, D = p.shape
    for t, n in ((delta_t, "delta_t"), (lam, "lambda")):
        _need_cuda(t, f"{fn}: {n}")
        if t.dtype != torch.float32 or t.device != p.device:
            raise ValueError(f"{fn}: {n} must be float32 on {p.device}")
    if delta_t.dim() != 2 or tuple(delta_t.shape) != (B, T) or (T > 1 and delta_t.stride(1) != 1):
        raise ValueError(f"{fn}: delta_t must be (B, T) = ({B}, {T}) with contiguous rows")
    if lam.dim() != 1 or lam.shape[0] != D or (D > 1 and lam.stride(0) != 1):
        raise ValueError(f"{fn}: lambda must be a contiguous (D,) vector")
    return delta_t.data_ptr(), (delta_t.stride(0) if B > 1 else T), lam.data_ptr()


def mingru_scan_decay(k: torch.Tensor, hx: torch.Tensor, h0: Optional[torch.Tensor],
                      delta_t: torch.Tensor, lam: torch.Tensor, log1p_delta: bool = False,
                      out: Optional[torch.Tensor] = None,
                      workspace: Optional[Workspace] = None) -> torch.Tensor:
    """minGRU with time decay: the state is gated by exp(-lam_d u_bt) at every
    token boundary (u = delta_t, or log1p(delta_t)); delta_t (B, T) and lam (D,)
    are float32 whatever the I/O dtype."""
    fn = "mingru_scan_decay"
    _seq(k, fn + ": k")
    _seq(hx, fn + ": hx")
    if k.shape != hx.shape or k.dtype != hx.dtype or k.device != hx.device:
        raise ValueError(f"{fn}: operands must share shape, dtype and device")
    dt = _dtype_code(k, fn)
    B, T, D = k.shape
    ip, ibs = _rows(h0, B, D, k, fn + ": initial state")
    gp, gbs, lp = _decay_operands(fn, k, delta_t, lam)
    if out is None:
        out = torch.empty_like(k)
    need = int(lib().sgr_workspace_size(_abi.SGR_OP_MINGRU, B, T, D, dt))
    wp, wn = 0, 0
    if need:
        ws = workspace if workspace is not None else default_workspace(k.device, need)
        wp, wn = ws.ptr, ws.nbytes
    with torch.cuda.device(k.device):
        code = lib().mingru_scan_decay(k.data_ptr(), hx.data_ptr(), ip, ibs, gp, gbs, lp,
                                       int(bool(log1p_delta)), out.data_ptr(), B, T, D, dt, wp, wn,
                                       _stream(k.device))
    check(fn, code)
    return out


def mingru_scan_decay_backward(k, hx, h0, delta_t, lam, h, dh, log1p_delta: bool = False,
                               want_dh0: bool = True, want_dlam: bool = True,
                               workspace: Optional[Workspace] = None):
    """(dk, dhx, dh0, dlam) through mingru_scan_decay for dL/dh = dh."""
    fn = "mingru_scan_decay_backward"
    for t, n in ((k, "k"), (hx, "hx"), (h, "h"), (dh, "dh")):
        _seq(t, f"{fn}: {n}")
        if t.shape != k.shape or t.dtype != k.dtype or t.device != k.device:
            raise ValueError(f"{fn}: {n} must match k's shape, dtype and device")
    dt = _dtype_code(k, fn)
    B, T, D = k.shape
    ip, ibs = _rows(h0, B, D, k, fn + ": initial state")
    gp, gbs, lp = _decay_operands(fn, k, delta_t, lam)
    dk, dhx = torch.empty_like(k), torch.empty_like(k)
    dh0 = torch.empty((B, D), dtype=k.dtype, device=k.device) if want_dh0 else None
    dlam = torch.empty((D,), dtype=torch.float32, device=k.device) if want_dlam else None
    need = int(lib().sgr_backward_workspace_size(_abi.SGR_OP_MINGRU, B, T, D, dt))
    wp, wn = 0, 0
    if need:
        ws = workspace if workspace is not None else default_workspace(k.device, need)
        wp, wn = ws.ptr, ws.nbytes
    with torch.cuda.device(k.device):
        code = lib().mingru_scan_decay_backward(
            k.data_ptr(), hx.data_ptr(), ip, ibs, gp, gbs, lp, int(bool(log1p_delta)), h.data_ptr(),
            dh.data_ptr(), dk.data_ptr(), dhx.data_ptr(), dh0.data_ptr() if dh0 is not None else 0, D,
            dlam.data_ptr() if dlam is not None else 0, B, T, D, dt, wp, wn, _stream(k.device))
    check(fn, code)
    return dk, dhx, dh0, dlam


def mingru_projected_scan(x: torch.Tensor, w: torch.Tensor, h0: Optional[torch.Tensor] = None,
                          out: Optional[torch.Tensor] = None,
                          workspace: Optional[Workspace] = None) -> torch.Tensor:
    """h (B, T, D) float32 = minGRU scan of k = x w[:D]^T, hx = x w[D:]^T, with
    the projection on the tensor cores in the same kernel (x (B, T, d_in) and
    w (2 D, d_in) bfloat16; D % 64 == 0, d_in % 64 == 0)."""
    fn = "mingru_projected_scan"
    _seq(x, fn + ": x")
    _need_cuda(w, fn + ": w")
    if x.dtype != torch.bfloat16 or w.dtype != torch.bfloat16 or w.device != x.device:
        raise ValueError(f"{fn}: x and w must be bfloat16 on one device")
    if w.dim() != 2 or w.shape[1] != x.shape[2] or w.shape[0] % 2 or not w.is_contiguous():
        raise ValueError(f"{fn}: w must be a contiguous (2 D, d_in) matrix")
    B, T, d_in = x.shape
    D = w.shape[0] // 2
    like = torch.empty(0, dtype=torch.float32, device=x.device)
    ip, ibs = _rows(h0, B, D, like, fn + ": h0")
    if out is None:
        out = torch.empty((B, T, D), dtype=torch.float32, device=x.device)
    elif tuple(out.shape) != (B, T, D) or out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError(f"{fn}: out must be a contiguous (B, T, D) float32 tensor")
    need = int(lib().sgr_projected_workspace_size(B, T, D))
    wp, wn = 0, 0
    if need:
        ws = workspace if workspace is not None else default_workspace(x.device, need)
        wp, wn = ws.ptr, ws.nbytes
    with torch.cuda.device(x.device):
        code = lib().mingru_projected_scan(x.data_ptr(), w.data_ptr(), ip, ibs, out.data_ptr(), B, T, D, d_in,
                                           wp, wn, _stream(x.device))
    check(fn, code)
    return out


def mingru_step(k_t: torch.Tensor, hx_t: torch.Tensor, h_prev: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One token: (B, D) rows in (any batch stride, contiguous along D), new
    state (B, D) out.  ``out`` may be ``h_prev`` for an in-place update."""
    for t, n in ((k_t, "k_t"), (hx_t, "hx_t")):
        _need_cuda(t, n)
        if t.dim() != 2:
            raise ValueError(f"mingru_step: {n} must be (B, D)")
    if k_t.shape != hx_t.shape or k_t.dtype != hx_t.dtype or k_t.device != hx_t.device:
        raise ValueError("mingru_step: k_t and hx_t must share shape, dtype and device")
    dt = _dtype_code(k_t, "mingru_step")
    B, D = k_t.shape
    kp, kbs = _rows(k_t, B, D, k_t, "k_t")
    hp, hbs = _rows(hx_t, B, D, k_t, "hx_t")
    pp, pbs = _rows(h_prev, B, D, k_t, "h_prev")
    if out is None:
        out = torch.empty((B, D), dtype=k_t.dtype, device=k_t.device)
    op, obs = _rows(out, B, D, k_t, "out")
    with torch.cuda.device(k_t.device):
        code = lib().mingru_step(kp, kbs, hp, hbs, pp, pbs, op, obs, B, D, dt, _stream(k_t.device))
    check("mingru_step", code)
    return out


def set_tile_override(channel_lanes: int = 0, rows_per_thread: int = 0) -> None:
    """Force the chunk shape of the scans (0, 0 restores the automatic choice)."""
    check("sgr_set_tile_override", lib().sgr_set_tile_override(channel_lanes, rows_per_thread))


def set_kernel_override(kernel: int = 0) -> None:
    """0 automatic, 1 tile kernel, 2 pipelined kernel, 3 pipelined with 15-warp
    blocks, 4 channel-sequential kernel (one warp per 32-channel group), 5 the
    same with each slot's rows split between half-warps, 6 two warps per
    32-channel group, 7 two warps per 64-channel group, two channels per lane
    (bf16), 8 four warps per 64-channel group (bf16; 2-8 where the fast path
    applies).  Gradients: 1 the tile
    kernel, 2 the pipelined gradient with 7-warp blocks (two per SM), 3 with
    15-warp blocks (one per SM), 4 the channel-sequential gradient."""
    check("sgr_set_kernel_override", lib().sgr_set_kernel_override(kernel))


def version() -> str:
    return lib().sgr_version().decode()
