"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

- the library loads and exports every function include/scan_gated_rnns.h declares;
- argument errors are reported before anything is enqueued;
- the tile plan's index arithmetic, replayed here for every block and thread of
  the benchmark and parity shapes, stays inside the buffers it addresses and
  covers every output element exactly once.
"""
import ctypes
import os
import re

import numpy as np
import pytest

from scan_gated_rnns_b200 import _abi
from scan_gated_rnns_b200.synth import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "scan_gated_rnns.h")

F32, BF16 = _abi.SGR_F32, _abi.SGR_BF16
MINGRU, MINMAX = _abi.SGR_OP_MINGRU, _abi.SGR_OP_MINMAX


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^SGR_API\s+[\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_three_operations():
    names = declared_functions()
    for n in ("mingru_scan", "mingru_step", "minmax_scan"):
        assert n in names


def test_every_declared_function_is_exported_and_typed():
    lib = _abi.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _abi.SIGNATURES, f"{name} has no ctypes signature"


def test_version_and_status_strings():
    assert "sm_100a" in _abi.lib().sgr_version().decode()
    for code in range(6):
        assert _abi.status_string(code)
    assert _abi.status_string(99) == "unknown status"


# ----------------------------------------------------- argument validation
# Fake device addresses: validation must reject these calls before touching
# CUDA.  The overlap checks need distinct non-null addresses, so these tests
# run only where no CUDA device is visible: should a check ever regress, the
# call then fails to launch (no device) instead of running a kernel on
# addresses that back nothing.
A, Bp, C = 0x10000000, 0x20000000, 0x30000000


def _device_visible() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:  # noqa: BLE001 - no torch: no device either
        return False


fake_addresses = pytest.mark.skipif(_device_visible(),
                                    reason="fake device addresses are only passed where no GPU is visible")


def scan(fn, *args):
    return getattr(_abi.lib(), fn)(*args)


@fake_addresses
@pytest.mark.parametrize("fn", ["mingru_scan", "minmax_scan"])
def test_scan_argument_errors(fn):
    E = _abi.SGR_ERR_INVALID_ARG
    # negative sizes / strides, unknown dtype
    assert scan(fn, A, Bp, None, 0, C, -1, 4, 4, F32, None, 0, None) == E
    assert scan(fn, A, Bp, None, 0, C, 1, -4, 4, F32, None, 0, None) == E
    assert scan(fn, A, Bp, 0x40000000, -1, C, 1, 4, 4, F32, None, 0, None) == E
    assert scan(fn, A, Bp, None, 0, C, 1, 4, 4, 7, None, 0, None) == E
    # null operands with data to move
    assert scan(fn, None, Bp, None, 0, C, 1, 4, 4, F32, None, 0, None) == E
    assert scan(fn, A, None, None, 0, C, 1, 4, 4, F32, None, 0, None) == E
    assert scan(fn, A, Bp, None, 0, None, 1, 4, 4, F32, None, 0, None) == E
    # output overlapping an input
    assert scan(fn, A, Bp, None, 0, A + 16, 1, 4, 4, F32, None, 0, None) == E
    assert scan(fn, A, Bp, C + 8, 4, C, 1, 4, 4, F32, None, 0, None) == E
    # empty shapes are no-ops, even with null pointers
    for shp in [(0, 4, 4), (2, 0, 4), (2, 4, 0)]:
        assert scan(fn, None, None, None, 0, None, *shp, F32, None, 0, None) == _abi.SGR_OK
    # a long sequence needs a workspace
    assert scan(fn, A, Bp, None, 0, C, 1, 1 << 16, 64, F32, None, 0, None) == _abi.SGR_ERR_WORKSPACE
    need = _abi.plan(MINGRU, 1, 1 << 16, 64, F32, True)["workspace_bytes"]
    assert 0 < need <= _abi.lib().sgr_workspace_size(MINGRU, 1, 1 << 16, 64, F32)
    assert scan(fn, A, Bp, None, 0, C, 1, 1 << 16, 64, F32, 0x50000000, need - 1, None) \
        == _abi.SGR_ERR_WORKSPACE
    assert scan(fn, A, Bp, None, 0, C, 1, 1 << 16, 64, F32, 0x50000008, need, None) \
        == _abi.SGR_ERR_WORKSPACE   # misaligned
    # byte counts that overflow int64
    assert scan(fn, A, Bp, None, 0, C, 1 << 40, 1 << 20, 1 << 10, F32, None, 0, None) \
        == _abi.SGR_ERR_UNSUPPORTED


@fake_addresses
def test_step_argument_errors():
    lib = _abi.lib()
    E = _abi.SGR_ERR_INVALID_ARG
    assert lib.mingru_step(A, 8, Bp, 8, None, 0, C, 8, 2, 8, 5, None) == E          # dtype
    assert lib.mingru_step(A, 8, Bp, 8, None, 0, C, 4, 2, 8, F32, None) == E        # out rows overlap
    assert lib.mingru_step(A, -8, Bp, 8, None, 0, C, 8, 2, 8, F32, None) == E       # stride
    assert lib.mingru_step(None, 8, Bp, 8, None, 0, C, 8, 2, 8, F32, None) == E
    assert lib.mingru_step(A, 8, Bp, 8, None, 0, A + 4, 8, 2, 8, F32, None) == E    # out on k
    assert lib.mingru_step(A, 8, Bp, 8, C + 4, 8, C, 8, 2, 8, F32, None) == E       # partial overlap
    assert lib.mingru_step(A, 8, Bp, 8, None, 0, C, 8, 0, 8, F32, None) == _abi.SGR_OK


def test_decayed_plan():
    # the decayed scan takes the plain scan's plan: wide batches the
    # channel-sequential kernel, otherwise the pipelined kernel with the
    # plain scan's rows per thread (4 fp32, 8 bf16) and block shape
    for B, T, D, dtype in ((16, 2048, 2048, F32), (24, 2048, 2048, BF16)):
        plain = _abi.plan(MINGRU, B, T, D, dtype, True)
        pl = _abi.plan(MINGRU, B, T, D, dtype, True, decay=True)
        assert pl["kernel"] == plain["kernel"] and pl["kernel"] in SEQ_KINDS, (B, T, D, dtype)
        assert pl["workspace_bytes"] == WS_HEADER
    # bf16 from 16 groups per SM: four warps per 64-channel group
    for B, want in ((16, _abi.KERNEL_SEQUENTIAL_PAIR), (20, _abi.KERNEL_SEQUENTIAL_QUAD),
                    (32, _abi.KERNEL_SEQUENTIAL_QUAD)):
        assert _abi.plan(MINGRU, B, 2048, 4096, BF16, True, decay=True)["kernel"] == want, B
    for B, T, D, dtype in ((8, 4096, 1024, BF16), (8, 4096, 1024, F32), (4, 8192, 512, BF16)):
        plain = _abi.plan(MINGRU, B, T, D, dtype, True)
        pl = _abi.plan(MINGRU, B, T, D, dtype, True, decay=True)
        assert pl["kernel"] in (_abi.KERNEL_PIPELINED, _abi.KERNEL_PIPELINED_WIDE), (B, T, D, dtype)
        assert pl["rows_per_thread"] == (4 if dtype == F32 else 8)
        assert (pl["kernel"], pl["warps"], pl["tile_rows"]) == (plain["kernel"], plain["warps"], plain["tile_rows"])
        assert pl["workspace_bytes"] <= _abi.lib().sgr_workspace_size(MINGRU, B, T, D, dtype)
    # small shapes: one launch per tile, as for the plain scan
    assert _abi.plan(MINGRU, 2, 1024, 512, F32, True, decay=True)["kernel"] == _abi.KERNEL_TILE
    # unaligned rows: the scalar tile kernel
    assert _abi.plan(MINGRU, 8, 4096, 1024, F32, False, decay=True)["kernel"] == _abi.KERNEL_TILE
    with pytest.raises(ValueError):
        _abi.plan(MINMAX, 8, 4096, 1024, F32, True, decay=True)
    lib = _abi.lib()
    assert lib.sgr_scan_plan_decay(8, 4096, 1024, 7, 1, None) == _abi.SGR_ERR_INVALID_ARG


def test_workspace_covers_the_decayed_plan():
    # the size covers the plain and the time-decayed plan of a shape: wide
    # batches need the header alone for both, narrower ones hand-off words
    lib = _abi.lib()
    for B, T, D, dtype in ((16, 2048, 2048, F32), (24, 2048, 2048, BF16), (8, 4096, 1024, BF16),
                           (1, 1 << 16, 64, F32)):
        need = lib.sgr_workspace_size(MINGRU, B, T, D, dtype)
        for decay in (False, True):
            for aligned in (True, False):
                assert _abi.plan(MINGRU, B, T, D, dtype, aligned, decay=decay)["workspace_bytes"] <= need


def test_workspace_size_and_hooks():
    lib = _abi.lib()
    assert lib.sgr_workspace_size(MINGRU, 2, 1, 512, F32) == WS_HEADER     # one chunk: the header
    assert lib.sgr_workspace_size(MINGRU, 0, 1, 512, F32) == 0             # empty shape
    assert lib.sgr_workspace_size(9, 2, 4096, 512, F32) == 0
    assert lib.sgr_workspace_size(MINGRU, 8, 4096, 1024, F32) > 0
    assert lib.sgr_set_tile_override(3, 0) == _abi.SGR_ERR_INVALID_ARG
    assert lib.sgr_set_tile_override(0, 3) == _abi.SGR_ERR_INVALID_ARG
    assert lib.sgr_set_drop_publish(-2) == _abi.SGR_ERR_INVALID_ARG
    assert lib.sgr_set_kernel_override(9) == _abi.SGR_ERR_INVALID_ARG
    assert lib.sgr_set_kernel_override(_abi.KERNEL_SEQUENTIAL_SPLIT) == _abi.SGR_OK
    assert lib.sgr_set_kernel_override(0) == _abi.SGR_OK
    assert lib.sgr_set_wait_limit(0) == _abi.SGR_OK
    assert lib.sgr_set_drop_publish(-1) == _abi.SGR_OK
    assert lib.sgr_workspace_init(None, 0, None) == _abi.SGR_OK
    assert lib.sgr_workspace_init(None, 64, None) == _abi.SGR_ERR_INVALID_ARG
    assert lib.sgr_workspace_status(None, 64, 0, None) == _abi.SGR_ERR_INVALID_ARG


# ----------------------------------------------------- index arithmetic
# The kernel's address formulas, replayed for every block and thread.

SEQ_ROWS = 16            # rows per load slot of the channel-sequential kernel
SEQ_KINDS = (_abi.KERNEL_SEQUENTIAL, _abi.KERNEL_SEQUENTIAL_SPLIT, _abi.KERNEL_SEQUENTIAL_PAIR,
             _abi.KERNEL_SEQUENTIAL_PAIR2, _abi.KERNEL_SEQUENTIAL_QUAD)
WS_HEADER = 256          # workspace header: status word at 0, chunk ticket at 64


def check_sequential_indices(pl, B, T, D, esz, check_cover):
    """The channel-sequential kernels: warp gw scans channel group gw % n_groups
    (32 channels; 16 when each slot's rows are split between the half-warps)
    of batch row gw // n_groups over the whole sequence, in slots of 16 rows
    loaded and stored as tensor-memory-accelerator boxes of CW channels x 16
    rows; lane l owns channel l % CW of the slot rows
    [(l // CW) R, (l // CW) R + R), R = 16 CW / 32.  With two warps per group
    (kernel 6) a block's warps w = 0, 1 take rows [32 i + 16 w, 32 i + 16 w + 16)
    of slot i, lane l channel l.  Kernel 7 (bf16): the same with groups of 64
    channels, lane l owning channels 2 l and 2 l + 1 (one 32-bit word of a
    128-byte row); kernel 8: kernel 7 with four warps per group, warp w taking
    rows [32 i + 8 w, 32 i + 8 w + 8) of slot i (boxes of 8 rows)."""
    V, CW = pl["channels_per_thread"], pl["tile_channels"]
    quad = pl["kernel"] == _abi.KERNEL_SEQUENTIAL_QUAD
    pair2 = pl["kernel"] == _abi.KERNEL_SEQUENTIAL_PAIR2 or quad
    pair = pl["kernel"] == _abi.KERNEL_SEQUENTIAL_PAIR or pair2
    split = 2 if pl["kernel"] == _abi.KERNEL_SEQUENTIAL_SPLIT else 1
    nw = 4 if quad else 2 if pair else 1                # warps per group
    rw = 32 // nw if pair else SEQ_ROWS                 # a warp's rows of a slot (box height)
    rb = CW * esz                                       # bytes of one operand row of a group
    if pair2:
        assert esz == 2 and V == 2 and CW == 64 and rb == 128
    else:
        assert V == 1 and CW == 32 // split and rb in (32, 64, 128)
    assert pl["vector_path"] and pl["channel_lanes"] * V == CW and pl["threads"] == 32 * pl["warps"]
    assert pl["warps"] == nw
    assert pl["rows_per_thread"] == (rw if pair else SEQ_ROWS // split)
    assert pl["n_chunks"] == 1 and pl["workspace_bytes"] == WS_HEADER and pl["tile_rows"] == T
    # a lane's elements of a slot stay inside its warp's rw rows of CW channels
    lane = np.arange(32)
    if pair2:
        off = lane * 4                                  # channels 2 l, 2 l + 1: one 32-bit word
        assert (off + (rw - 1) * rb + 4 <= rw * rb).all() and (off % 4 == 0).all()
        assert len(set(off.tolist())) == 32
    else:
        off = (lane // CW) * pl["rows_per_thread"] * rb + (lane % CW) * esz
        assert (off + (pl["rows_per_thread"] - 1) * rb + esz <= SEQ_ROWS * rb).all()
        assert len(set(zip(lane % CW, lane // CW))) == 32   # no two lanes share an element
    n_groups = -(-D // CW)
    assert pl["n_channel_tiles"] == n_groups and pl["n_chains"] == B * n_groups
    assert pl["n_tiles"] == pl["n_chains"] < 2 ** 31
    assert 2 <= pl["stages"] <= 8
    if pair:
        assert pl["stages"] == 2                        # the pair kernels keep two slots per warp
    # the warps' rings, staging buffers and mbarriers fit their block's shared memory
    S = pl["stages"]
    if pair:
        warp_bytes = -(-(S * 2 * rw * rb + rw * rb + S * 8) // 128) * 128
        block_bytes = nw * warp_bytes + 2 * nw * 32 * (16 if pair2 else 8)   # + the pairs exchanged per slot
    else:
        block_bytes = -(-(S * 2 * SEQ_ROWS * rb + 2 * SEQ_ROWS * rb + S * 8) // 128) * 128
    assert block_bytes <= pl["smem_bytes"] <= 227 * 1024
    assert (D * esz) % 16 == 0 and T < 2 ** 31 and B < 2 ** 31
    gw = np.arange(pl["n_chains"], dtype=np.int64)
    b, grp = gw // n_groups, gw % n_groups
    x0 = grp * CW
    assert ((x0 * esz) % 16 == 0).all()                 # box x coordinate 16-byte aligned
    assert (x0 < D).all() and (b < B).all()
    slot_rows = 2 * SEQ_ROWS if pair else SEQ_ROWS
    n_slots = -(-T // slot_rows)
    assert n_slots * slot_rows < 2 ** 31                # row coordinates are 32-bit
    if check_cover:
        # the store boxes, clipped to the tensor, write every element exactly once
        # (a pair warp's box that would start past T is not stored)
        cover = np.zeros((B, max(T, 1), D), dtype=np.int32)
        for w in range(len(gw)):
            for i in range(n_slots):
                for y0 in ([i * slot_rows + rw * v for v in range(nw)] if pair else [i * SEQ_ROWS]):
                    if y0 < T:
                        cover[b[w], y0:min(T, y0 + rw), x0[w]:min(D, x0[w] + CW)] += 1
        assert (cover[:, :T] == 1).all(), "every output element is written exactly once"


def check_plan_indices(B, T, D, dtype, aligned, check_cover, op=MINGRU):
    pl = _abi.plan(op, B, T, D, dtype, aligned)
    esz = 4 if dtype == F32 else 2
    if pl["kernel"] in SEQ_KINDS:
        check_sequential_indices(pl, B, T, D, esz, check_cover)
        return
    V, cg, R, W = pl["channels_per_thread"], pl["channel_lanes"], pl["rows_per_thread"], pl["warps"]
    J = 32 // cg
    TR, TC = pl["tile_rows"], pl["tile_channels"]
    n_dt, n_chains, n_chunks, n_tiles = pl["n_channel_tiles"], pl["n_chains"], pl["n_chunks"], pl["n_tiles"]
    assert TR == W * J * R and TC == cg * V and TC % 32 == 0
    assert n_dt == -(-D // TC) and n_chains == B * n_dt and n_chunks == -(-T // TR)
    assert n_tiles == n_chains * n_chunks and n_tiles < 2 ** 31
    assert pl["threads"] == (W + 1) * 32
    if pl["kernel"] in (_abi.KERNEL_PIPELINED, _abi.KERNEL_PIPELINED_WIDE):
        # persistent blocks: lane l owns channels l V.., warp w owns rows w R..
        assert pl["vector_path"] and cg * V * esz == 128 and V == 4 and pl["stages"] >= 2
        # tensor-memory-accelerator boxes of TC x TR x 1: inner extent a multiple of
        # 16 bytes, every box dimension <= 256, the x coordinate (dt TC) 16-byte aligned
        assert (TC * esz) % 16 == 0 and TC <= 256 and TR <= 256
        assert (D * esz) % 16 == 0 and (T * D * esz) % 16 == 0
        assert pl["threads"] % 128 == 0      # whole warps per SM sub-partition
        per_sm = 2 if pl["kernel"] == _abi.KERNEL_PIPELINED else 1
        assert pl["smem_bytes"] <= 227 * 1024 // per_sm
    if pl["vector_path"]:
        assert aligned and D % V == 0 and V * esz in (8, 16)
    # the kernels divide tile -> (chunk, chain) -> (b, dt) by multiply-high,
    # add and shift with the host's constants: exact for every tile index
    ti = np.arange(n_tiles, dtype=np.uint64)
    fd = lambda n, m, s: ((n * np.uint64(m)) >> np.uint64(32)) + n >> np.uint64(s)
    cq = fd(ti, pl["div_chains_m"], pl["div_chains_s"])
    assert (cq == ti // np.uint64(n_chains)).all()
    ch = np.arange(n_chains, dtype=np.uint64)
    assert (fd(ch, pl["div_dt_m"], pl["div_dt_s"]) == ch // np.uint64(n_dt)).all()
    # every (tile, warp, lane) piece, whichever block processes the tile
    tile = np.arange(n_tiles, dtype=np.int64)[:, None, None]
    warp = np.arange(W, dtype=np.int64)[None, :, None]
    lane = np.arange(32, dtype=np.int64)[None, None, :]
    chain, c = tile % n_chains, tile // n_chains
    b, dt = chain // n_dt, chain % n_dt
    g, j = lane % cg, lane // cg
    d0 = dt * TC + g * V
    row0 = c * TR + (warp * J + j) * R
    N = B * T * D
    cover = np.zeros(N, dtype=np.int32) if check_cover else None
    for r in range(R):
        t = row0 + r
        valid = (d0 < D) & (t < T)
        idx = ((b * T + t) * D + d0)[np.broadcast_to(valid, np.broadcast_shapes(valid.shape, d0.shape))]
        if idx.size:
            assert idx.min() >= 0 and idx.max() + V <= N
            dv = np.broadcast_to(d0, valid.shape)[valid]
            assert (dv + V <= D).all()
            if pl["vector_path"]:
                assert ((idx * esz) % (V * esz) == 0).all()
            if check_cover:
                for v in range(V):
                    np.add.at(cover, idx + v, 1)
    if check_cover:
        assert (cover == 1).all(), "every output element is written exactly once"
    # carry warp: lane l owns channels [l CV, l CV + CV); hand-off words inside the workspace
    CV = TC // 32
    assert (np.arange(32) * CV + CV - 1 < TC).all()
    if n_chunks > 1:
        # hand-off words after the header (status word, chunk ticket)
        assert pl["off_words"] >= WS_HEADER and pl["off_words"] % 8 == 0
        assert pl["off_words"] + 8 * 3 * TC * n_tiles <= pl["workspace_bytes"]
        assert _abi.lib().sgr_workspace_size(op, B, T, D, dtype) >= pl["workspace_bytes"]
    else:
        assert pl["workspace_bytes"] == WS_HEADER


SMALL_SHAPES = [(2, 1024, 512), (3, 1000, 96), (1, 777, 36), (2, 300, 7), (1, 1, 1), (5, 1, 64),
                (1, 4097, 32), (2, 129, 40), (4, 63, 8), (1, 2000, 1)]


@pytest.mark.parametrize("shape", SMALL_SHAPES)
@pytest.mark.parametrize("dtype", [F32, BF16])
@pytest.mark.parametrize("aligned", [True, False])
@pytest.mark.parametrize("override", [(0, 0, 0), (1, 0, 1), (1, 0, 2), (1, 0, 4), (1, 0, 8),
                                      (2, 0, 2), (2, 0, 4), (2, 0, 8), (3, 0, 2), (3, 0, 4),
                                      (3, 0, 8), (4, 0, 0), (5, 0, 0), (6, 0, 0), (7, 0, 0),
                                      (8, 0, 0)])
def test_plan_indices_small(shape, dtype, aligned, override):
    lib = _abi.lib()
    assert lib.sgr_set_kernel_override(override[0]) == 0
    assert lib.sgr_set_tile_override(*override[1:]) == 0
    try:
        check_plan_indices(*shape, dtype, aligned, check_cover=True)
    finally:
        lib.sgr_set_tile_override(0, 0)
        lib.sgr_set_kernel_override(0)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_plan_indices_workloads(name):
    w = WORKLOADS[name]
    op = MINGRU if w.op == "mingru" else _abi.SGR_OP_MINMAX
    check_plan_indices(w.B, w.T, w.D, F32 if w.dtype == "f32" else BF16, True, check_cover=False, op=op)


# ------------------------------------------------------- host-buffer scans

@fake_addresses
@pytest.mark.parametrize("fn", ["mingru_scan_host", "minmax_scan_host"])
def test_host_scan_argument_errors(fn):
    E = _abi.SGR_ERR_INVALID_ARG

    def call(p, q, init, ibs, out, B, T, D, dt=F32, chunks=0):
        return scan(fn, p, q, init, ibs, out, B, T, D, dt, chunks, None, 0, None)

    assert call(A, Bp, None, 0, C, -1, 4, 4) == E
    assert call(A, Bp, None, 0, C, 1, 4, 4, dt=7) == E
    assert call(A, Bp, None, 0, C, 1, 4, 4, chunks=-2) == E
    assert call(A, Bp, 0x40000000, -1, C, 1, 4, 4) == E
    assert call(None, Bp, None, 0, C, 1, 4, 4) == E
    assert call(A, Bp, None, 0, A + 16, 1, 4, 4) == E           # output on an input
    assert call(A, Bp, C + 8, 4, C, 1, 4, 4) == E               # output on the state
    for shp in [(0, 4, 4), (2, 0, 4), (2, 4, 0)]:
        assert call(None, None, None, 0, None, *shp) == _abi.SGR_OK
    assert call(A, Bp, None, 0, C, 1 << 40, 1 << 20, 1 << 10) == _abi.SGR_ERR_UNSUPPORTED


def test_host_staging_size():
    lib = _abi.lib()
    size = lambda B, T, D, dt=F32, chunks=0, op=MINGRU: lib.sgr_host_staging_size(op, B, T, D, dt, chunks)
    assert size(0, 4, 4) == 0 and size(1, 4, 4, dt=9) == 0 and size(1, 4, 4, chunks=-1) == 0
    assert size(1, 4, 4, op=5) == 0
    B, T, D = 8, 4096, 1024
    whole = B * T * D * 4
    # one slice: two sets of (two operands + output) of the whole tensor, plus state and workspace
    assert size(B, T, D, chunks=1) >= 6 * whole + B * D * 4
    prev = None
    for n in (1, 2, 3, 8, 64, T):
        s = size(B, T, D, chunks=n)
        tc = -(-T // n)
        assert s >= 6 * B * tc * D * 4
        if prev is not None:
            assert s <= prev
        prev = s
    assert size(B, T, D, chunks=T) == size(B, T, D, chunks=10 * T)    # at most one row per slice
    # automatic slices: n = round(sqrt(input MiB / 4.6)), 7 for these 256 MiB of
    # inputs; staging stays far below the tensor
    auto = size(B, T, D)
    assert auto == size(B, T, D, chunks=7) and auto < 6 * whole // 4
    assert size(2, 5, 3, op=MINMAX, chunks=2) > 0


# ------------------------------------------------------------- gradients

@fake_addresses
@pytest.mark.parametrize("fn", ["mingru_scan_backward", "minmax_scan_backward"])
def test_backward_argument_errors(fn):
    E = _abi.SGR_ERR_INVALID_ARG
    G, O0, O1, DI = 0x60000000, 0x70000000, 0x80000000, 0x90000000

    def call(p=A, q=Bp, init=None, ibs=0, fwd=C, gy=G, o0=O0, o1=O1, di=None, dbs=0,
             B=2, T=4, D=8, dt=F32, ws=None, wn=0):
        return scan(fn, p, q, init, ibs, fwd, gy, o0, o1, di, dbs, B, T, D, dt, ws, wn, None)

    assert call(B=-1) == E
    assert call(dt=7) == E
    assert call(ibs=-1) == E
    assert call(dbs=-8) == E
    for kw in ({"p": None}, {"q": None}, {"fwd": None}, {"gy": None}, {"o0": None}, {"o1": None}):
        assert call(**kw) == E
    assert call(o0=A + 64) == E                   # output on an input
    assert call(o1=G) == E
    assert call(o1=O0 + 16) == E                  # the two outputs overlap
    assert call(di=O1 + 32, dbs=8) == E           # initial-state gradient on an output
    assert call(di=DI, dbs=4) == E                # its rows would overlap each other
    for shp in [(0, 4, 4), (2, 4, 0)]:
        B, T, D = shp
        assert call(p=None, q=None, fwd=None, gy=None, o0=None, o1=None, B=B, T=T, D=D) == _abi.SGR_OK
    assert call(B=1 << 40, T=1 << 20, D=1 << 10) == _abi.SGR_ERR_UNSUPPORTED
    # long sequences need a workspace
    assert call(B=1, T=1 << 16, D=64) == _abi.SGR_ERR_WORKSPACE
    need = _abi.lib().sgr_backward_workspace_size(MINGRU, 1, 1 << 16, 64, F32)
    assert need > 0
    assert call(B=1, T=1 << 16, D=64, ws=0x50000000, wn=256) == _abi.SGR_ERR_WORKSPACE
    assert call(B=1, T=1 << 16, D=64, ws=0x50000008, wn=need) == _abi.SGR_ERR_WORKSPACE   # misaligned


@pytest.mark.parametrize("shape", [(2, 1000, 96), (1, 777, 36), (3, 129, 40), (1, 1, 1), (2, 300, 7)])
@pytest.mark.parametrize("dtype", [F32, BF16])
@pytest.mark.parametrize("aligned", [True, False])
def test_backward_plan_reverse_indices(shape, dtype, aligned):
    """Replay the gradient kernel's reverse-time indexing: every (b, t, d) is
    written exactly once, the state row read (t - 1) is in range or the
    initial state, and exactly one thread per channel ends at time row 0."""
    B, T, D = shape
    pl = _abi.plan(MINGRU, B, T, D, dtype, aligned)   # forward plan: only for V / layout
    lib = _abi.lib()
    assert lib.sgr_set_kernel_override(1) == 0       # the tile plan the gradient kernel uses
    try:
        pl = _abi.plan(MINGRU, B, T, D, dtype, aligned)
    finally:
        lib.sgr_set_kernel_override(0)
    V, cg, R, W = pl["channels_per_thread"], pl["channel_lanes"], pl["rows_per_thread"], pl["warps"]
    while R > 1 and R * V > 16:   # the gradient kernel's cap on elements per thread
        R //= 2
    J = 32 // cg
    TR, TC = W * J * R, cg * V
    n_dt = -(-D // TC)
    n_chains = B * n_dt
    n_chunks = -(-T // TR)
    assert R * V <= 16
    cover = np.zeros((B, T, D), dtype=np.int32)
    ends_at_zero = np.zeros((B, D), dtype=np.int32)
    for tile in range(n_chains * n_chunks):
        c, chain = divmod(tile, n_chains)
        b, dt = divmod(chain, n_dt)
        ct = n_chunks - 1 - c
        for warp in range(W):
            for lane in range(32):
                g, j = lane % cg, lane // cg
                d0 = dt * TC + g * V
                if d0 >= D:
                    continue
                top = ct * TR + TR - 1 - (warp * J + j) * R
                for r in range(R):
                    t = top - r
                    assert t >= 0
                    if t < T:
                        cover[b, t, d0:d0 + V] += 1
                        assert t - 1 >= -1
                if top - (R - 1) == 0:
                    ends_at_zero[b, d0:d0 + V] += 1
    assert (cover == 1).all()
    assert (ends_at_zero == 1).all()


@fake_addresses
def test_decay_argument_errors():
    lib = _abi.lib()
    E = _abi.SGR_ERR_INVALID_ARG
    G, L = 0x60000000, 0x70000000

    def call(dt=G, dbs=4, lam=L, B=2, T=4, D=8):
        return lib.mingru_scan_decay(A, Bp, None, 0, dt, dbs, lam, 0, C, B, T, D, F32, None, 0, None)

    assert call(dt=None) == E
    assert call(lam=None) == E
    assert call(dbs=-1) == E
    assert call(dbs=3) == E              # gap rows of a (B, T) array would overlap
    assert call(B=0) == _abi.SGR_OK
    db = lib.mingru_scan_decay_backward
    args = (A, Bp, None, 0, G, 3, L, 0, C, 0x80000000, 0x90000000, 0xA0000000, None, 0, 0xB0000000,
            2, 4, 8, F32, None, 0, None)
    assert db(*args) == E               # overlapping gap rows

    # outputs sharing memory with the gaps or the rates, and dL/dlambda
    # sharing memory with any operand: refused before anything is queued
    span = 2 * 4 * 8 * 4                                       # one (2, 4, 8) fp32 tensor
    assert call(dt=C + 16) == E
    assert call(lam=C + span - 4) == E
    big = dict(B=2, T=1 << 16, D=64, dbs=1 << 16)              # chunked: needs a workspace
    assert call(dt=C + 2 * (1 << 16) * 64 * 4, **big) == _abi.SGR_ERR_WORKSPACE   # adjacent, no overlap
    ok = list(args)
    ok[5] = 4                                                  # gap rows of 4: no overlap among them
    ok[13] = 8                                                 # dh0 rows of D (used when dh0 is set)
    for i, v in ((14, A + 4), (14, G + 4), (14, L + 4), (14, 0x90000000 + 4), (14, C + 4),
                 (10, L), (10, G + 8), (11, L + 16), (12, G)):
        bad = list(ok)
        bad[i] = v
        assert db(*bad) == E, (i, hex(v))
    ok[15:18] = [2, 1 << 16, 64]
    ok[5] = 1 << 16
    assert db(*ok) == _abi.SGR_ERR_WORKSPACE                   # distinct buffers pass the checks


@fake_addresses
def test_summary_and_combine_argument_errors():
    lib = _abi.lib()
    E = _abi.SGR_ERR_INVALID_ARG
    P, W = 0x60000000, 0x70000000
    need = lib.sgr_summary_workspace_size(2, 100, 64, F32)
    assert need > 0 and lib.sgr_summary_workspace_size(0, 100, 64, F32) == 0
    s = lambda *a: lib.sgr_scan_summary(*a)   # noqa: E731
    assert s(MINGRU, A, Bp, -1, 100, 64, F32, P, W, need, None) == E
    assert s(7, A, Bp, 2, 100, 64, F32, P, W, need, None) == E
    assert s(_abi.SGR_OP_MINGRU_LOG, A, Bp, 2, 100, 64, F32, P, W, need, None) == E   # linear pairs only
    assert s(MINGRU, A, Bp, 2, 100, 64, 9, P, W, need, None) == E
    assert s(MINGRU, A, Bp, 2, 100, 64, F32, None, W, need, None) == E
    assert s(MINGRU, None, Bp, 2, 100, 64, F32, P, W, need, None) == E
    assert s(MINGRU, A, Bp, 2, 100, 64, F32, A + 64, W, need, None) == E      # pairs on an input
    assert s(MINGRU, A, Bp, 2, 100, 64, F32, P, None, 0, None) == _abi.SGR_ERR_WORKSPACE
    # the size covers both the aligned (warp per segment) and the unaligned
    # plan; 256 bytes, less than either needs, is rejected for both alignments
    assert s(MINGRU, A, Bp, 2, 100, 64, F32, P, W, 256, None) == _abi.SGR_ERR_WORKSPACE
    assert s(MINGRU, A + 4, Bp, 2, 100, 64, F32, P, W, 256, None) == _abi.SGR_ERR_WORKSPACE
    assert s(MINGRU, A, Bp, 2, 100, 64, F32, P, P, need, None) == E           # workspace on the pairs
    assert s(MINGRU, A, Bp, 0, 100, 64, F32, None, None, 0, None) == _abi.SGR_OK
    c = lambda *a: lib.sgr_combine_summaries(*a)   # noqa: E731
    assert c(MINGRU, P, -1, None, 0, C, 64, 2, 64, F32, None) == E
    assert c(MINGRU, None, 1, None, 0, C, 64, 2, 64, F32, None) == E          # pairs needed for rank > 0
    assert c(MINGRU, P, 1, None, 0, C, 32, 2, 64, F32, None) == E             # out rows overlap
    assert c(MINGRU, P, 1, None, 0, P + 8, 64, 2, 64, F32, None) == E         # out on the pairs
    assert c(MINGRU, P, 1, C + 4, 64, C, 64, 2, 64, F32, None) == E           # out partly on init
    assert c(MINGRU, P, 1, None, 0, None, 64, 0, 64, F32, None) == _abi.SGR_OK
    assert c(_abi.SGR_OP_MINGRU_LOG, P, 1, None, 0, C, 64, 2, 64, F32, None) == E


@fake_addresses
def test_projected_scan_argument_errors():
    lib = _abi.lib()
    X, W, H, WS = 0x10000000, 0x20000000, 0x30000000, 0x40000000

    def call(x=X, w=W, h0=None, hbs=0, h=H, B=2, T=10, D=128, d=64, ws=WS, wn=1 << 20):
        return lib.mingru_projected_scan(x, w, h0, hbs, h, B, T, D, d, ws, wn, None)

    E = _abi.SGR_ERR_INVALID_ARG
    assert call(B=-1) == E
    assert call(x=None) == E
    assert call(x=X + 8) == E                    # x must be 16-byte aligned (tensor map)
    assert call(D=96) == _abi.SGR_ERR_UNSUPPORTED
    assert call(d=48) == _abi.SGR_ERR_UNSUPPORTED
    assert call(h=X + 64) == E                   # output on x
    assert call(ws=None, wn=0) == _abi.SGR_ERR_WORKSPACE
    assert call(wn=lib.sgr_projected_workspace_size(2, 10, 128) - 1) == _abi.SGR_ERR_WORKSPACE
    assert call(B=0) == _abi.SGR_OK
    assert lib.sgr_projected_workspace_size(2, 10, 96) == 0


def test_backward_kernel_choice():
    """The gradient walks whole sequences per warp (kernel 4) from 5 warps of
    32 channels per SM, on aligned vector-width rows; below that, on aligned
    vector-width rows, the pipelined gradient (2) once it has two tiles per
    block; otherwise the tile kernel (1)."""
    lib = _abi.lib()
    assert lib.sgr_backward_kernel(MINGRU, 16, 2048, 4096, BF16, 1) == 4     # 2048 groups
    assert lib.sgr_backward_kernel(MINGRU, 8, 2048, 4096, BF16, 1) == 4      # 1024 groups
    assert lib.sgr_backward_kernel(MINGRU, 4, 2048, 4096, BF16, 1) == 2      # 512 groups
    assert lib.sgr_backward_kernel(MINGRU, 2, 2048, 4096, BF16, 1) == 2      # 256 groups, 2304 tiles
    assert lib.sgr_backward_kernel(MINGRU, 8, 4096, 1024, F32, 1) == 2       # 256 groups, 8960 tiles
    assert lib.sgr_backward_kernel(_abi.SGR_OP_MINMAX, 4, 8192, 768, F32, 1) == 2
    assert lib.sgr_backward_kernel(MINGRU, 2, 1024, 512, F32, 1) == 1       # 352 tiles of 96 rows, 288 of 120
    assert lib.sgr_backward_kernel(MINGRU, 8, 4096, 1024, F32, 0) == 1       # unaligned
    assert lib.sgr_backward_kernel(MINGRU, 16, 2048, 4096, BF16, 0) == 1     # unaligned
    assert lib.sgr_backward_kernel(MINGRU, 16, 2048, 4100, BF16, 1) == 1     # D not a vector multiple
    assert lib.sgr_backward_kernel(9, 16, 2048, 4096, BF16, 1) == 0
    assert lib.sgr_set_kernel_override(4) == 0
    try:
        assert lib.sgr_backward_kernel(MINGRU, 1, 10, 32, F32, 1) == 4
        assert lib.sgr_backward_kernel(MINGRU, 1, 10, 36, F32, 1) == 4       # partial group, aligned rows
        assert lib.sgr_backward_kernel(MINGRU, 1, 10, 6, F32, 1) == 1        # rows not 16-byte multiples
    finally:
        lib.sgr_set_kernel_override(0)


def test_log_space_plan():
    """mingru_scan_log runs the chunked kernels at any batch width: its plan is
    never channel-sequential, and its workspace size covers it where the
    linear scan of a wide batch needs only the header.  Gradients, summaries
    and the decayed form do not take it."""
    lib = _abi.lib()
    LOG = _abi.SGR_OP_MINGRU_LOG
    for B, T, D, dt in [(16, 2048, 4096, BF16), (8, 4096, 1024, F32), (2, 1000, 96, F32), (64, 512, 2048, F32)]:
        for aligned in (True, False):
            pl = _abi.plan(LOG, B, T, D, dt, aligned)
            assert pl["kernel"] in (_abi.KERNEL_TILE, _abi.KERNEL_PIPELINED, _abi.KERNEL_PIPELINED_WIDE)
            assert lib.sgr_workspace_size(LOG, B, T, D, dt) >= pl["workspace_bytes"]
    assert _abi.plan(MINGRU, 16, 2048, 4096, BF16)["workspace_bytes"] == WS_HEADER
    assert lib.sgr_workspace_size(LOG, 16, 2048, 4096, BF16) > WS_HEADER
    assert lib.sgr_backward_workspace_size(LOG, 8, 4096, 1024, F32) == 0
    assert lib.sgr_backward_kernel(LOG, 8, 4096, 1024, F32, 1) == 0


@fake_addresses
def test_log_space_argument_errors():
    E = _abi.SGR_ERR_INVALID_ARG
    fn = "mingru_scan_log"
    assert scan(fn, A, Bp, None, 0, C, -1, 4, 4, F32, None, 0, None) == E
    assert scan(fn, None, Bp, None, 0, C, 1, 4, 4, F32, None, 0, None) == E
    assert scan(fn, A, Bp, None, 0, A + 16, 1, 4, 4, F32, None, 0, None) == E
    for shp in [(0, 4, 4), (2, 0, 4), (2, 4, 0)]:
        assert scan(fn, None, None, None, 0, None, *shp, F32, None, 0, None) == _abi.SGR_OK
    # a wide batch: the linear scan's header-only workspace is too small here
    assert scan(fn, A, Bp, None, 0, C, 16, 2048, 4096, BF16, 0x50000000, WS_HEADER, None) \
        == _abi.SGR_ERR_WORKSPACE


def test_bf16_channel_sequential_kind_choice():
    # B x 2048 x 4096 bf16 (B x 0.86 groups of 32 channels per SM): the minGRU
    # takes two warps per 32 channels below 16 groups per SM, four warps per
    # 64 channels up to 24, two per 64 channels above; MinMax four per 64
    # channels throughout; fp32 never the 64-channel forms
    for B, want in ((8, _abi.KERNEL_SEQUENTIAL_PAIR), (16, _abi.KERNEL_SEQUENTIAL_PAIR),
                    (20, _abi.KERNEL_SEQUENTIAL_QUAD), (24, _abi.KERNEL_SEQUENTIAL_QUAD),
                    (28, _abi.KERNEL_SEQUENTIAL_PAIR2), (32, _abi.KERNEL_SEQUENTIAL_PAIR2)):
        assert _abi.plan(MINGRU, B, 2048, 4096, BF16, True)["kernel"] == want, B
    for B in (8, 16, 32):
        assert _abi.plan(_abi.SGR_OP_MINMAX, B, 2048, 4096, BF16, True)["kernel"] == _abi.KERNEL_SEQUENTIAL_QUAD, B
    for B in (8, 16, 32):
        assert _abi.plan(MINGRU, B, 2048, 4096, F32, True)["kernel"] in (_abi.KERNEL_SEQUENTIAL,
                                                                          _abi.KERNEL_SEQUENTIAL_PAIR)
        assert _abi.plan(_abi.SGR_OP_MINMAX, B, 2048, 4096, F32, True)["kernel"] in (_abi.KERNEL_SEQUENTIAL,
                                                                                    _abi.KERNEL_SEQUENTIAL_PAIR)


def test_minmax_plans_take_the_long_tiles():
    """MinMax, next to no arithmetic per element, takes the 15-warp pipelined
    blocks wherever they still give every SM 4 tiles; minGRU on the same
    shape keeps the 7-warp blocks."""
    assert _abi.plan(_abi.SGR_OP_MINMAX, 4, 8192, 768, F32, True)["kernel"] == _abi.KERNEL_PIPELINED_WIDE
    assert _abi.plan(MINGRU, 4, 8192, 768, F32, True)["kernel"] == _abi.KERNEL_PIPELINED
    lib = _abi.lib()
    # the size query covers this plan (and the unaligned one)
    assert lib.sgr_workspace_size(_abi.SGR_OP_MINMAX, 4, 8192, 768, F32) >= \
        _abi.plan(_abi.SGR_OP_MINMAX, 4, 8192, 768, F32, True)["workspace_bytes"] > 0


@pytest.mark.parametrize("shape", [(2, 1000, 96), (1, 3001, 40), (1, 121, 64), (2, 7, 32), (3, 250, 160),
                                   (8, 4096, 1024)])
@pytest.mark.parametrize("dtype", [F32, BF16])
@pytest.mark.parametrize("override,W", [(2, 7), (3, 15)])
def test_pipelined_backward_indices(shape, dtype, override, W):
    """The pipelined gradient (persistent blocks, four copy boxes per tile):
    tiles numbered chain-fastest in processing order, processing chunk c
    covering time chunk n_chunks - 1 - c; boxes of TC x TR at (dt TC, ct TR, b),
    the forward output's one row earlier; lane (g, j) of warp w owns channels
    [g V, g V + V) of processing rows [(w J + j) R, (w J + j) R + R), processing
    row rho at slot row TR - 1 - rho.  Every slot row read is inside the slot,
    every (b, t, d) is written exactly once, exactly one thread per channel
    ends at time row 0, and the workspace covers the hand-off words.
    Override 2 takes blocks of 7 data warps (two per SM), 3 of 15 (one)."""
    B, T, D = shape
    esz = 4 if dtype == F32 else 2
    if D % (16 // esz):
        pytest.skip("vector rows only")
    lib = _abi.lib()
    assert lib.sgr_set_kernel_override(override) == 0
    try:
        assert lib.sgr_backward_kernel(MINGRU, B, T, D, dtype, 1) == 2
        need = lib.sgr_backward_workspace_size(MINGRU, B, T, D, dtype)
    finally:
        lib.sgr_set_kernel_override(0)
    cg, V = (8 if dtype == F32 else 16), 4
    R = 2 if dtype == F32 else 4
    J = 32 // cg
    TC, TR = cg * V, W * J * R
    assert TR == 8 * W and (TC * esz) % 16 == 0 and TC <= 256 and TR <= 256
    assert TR % 4 == 0                       # the decay gaps' box starts at ct TR: a 16-byte multiple
    n_dt = -(-D // TC)
    n_chains, n_chunks = B * n_dt, -(-T // TR)
    n_tiles = n_chains * n_chunks
    assert n_tiles < 2 ** 31 and n_chunks * TR < 2 ** 31
    if n_chunks > 1:
        assert need >= WS_HEADER + 8 * 3 * TC * n_tiles
    # a slot: four operand boxes, then (decay) TC rates and TR gaps; 3 slots
    slot = -(-(4 * TR * TC * esz + (TR + TC) * 4) // 128) * 128
    smem = 3 * slot + 3 * 8 + 3 * 4 + 16 + 2 * W * TC * 8 + 2 * TC * 8 + 2 * TC * 4 + 2 * TC * 4 + 16
    assert smem * (2 if W == 7 else 1) <= 228 * 1024 - 2 * 1024   # blocks per SM, 1 KB reserved each
    tile = np.arange(n_tiles, dtype=np.int64)[:, None, None]
    warp = np.arange(W, dtype=np.int64)[None, :, None]
    lane = np.arange(32, dtype=np.int64)[None, None, :]
    c, chain = tile // n_chains, tile % n_chains
    b, dt = chain // n_dt, chain % n_dt
    ct = n_chunks - 1 - c
    assert (ct * TR - 1 >= -1).all()         # the forward output's box starts at row -1 at the earliest
    g, j = lane % cg, lane // cg
    d0 = dt * TC + g * V
    rho0 = (warp * J + j) * R
    top = ct * TR + TR - 1 - rho0
    assert ((TR - 1 - rho0 - (R - 1)) >= 0).all() and ((TR - 1 - rho0) < TR).all()
    ends = (top - (R - 1) == 0) & (d0 < D)
    cnt0 = np.zeros((B, D), dtype=np.int32)
    bb, dd = np.broadcast_to(b, ends.shape)[ends], np.broadcast_to(d0, ends.shape)[ends]
    for v in range(V):
        np.add.at(cnt0, (bb, dd + v), 1)
    assert (cnt0 == 1).all(), "one thread per channel ends at time row 0"
    if B * T * D <= 1 << 22:
        cover = np.zeros((B, T, D), dtype=np.int32)
        for r in range(R):
            t = top - r
            ok = (t < T) & (d0 < D)
            tt = np.broadcast_to(t, ok.shape)[ok]
            b2, d2 = np.broadcast_to(b, ok.shape)[ok], np.broadcast_to(d0, ok.shape)[ok]
            assert (tt >= 0).all()
            for v in range(V):
                np.add.at(cover, (b2, tt, d2 + v), 1)
        assert (cover == 1).all(), "every element's gradient is written exactly once"


@pytest.mark.parametrize("shape", [(8, 4096, 1024), (4, 8192, 768), (1, 131072, 512), (3, 2501, 640),
                                   (3, 2501, 160)])
def test_fp32_gradient_pair_plan(shape):
    """The fp32 gradients' automatic plan where it gives every block two
    tiles (the decayed gradient at any chain count, the plain ones below 1.5
    chains of 32 channels per SM): blocks of 6 data warps + 1 carry warp, two
    per SM, 4 rows per thread (96-row tiles) and a 2-slot ring.  Two blocks' shared memory (with
    the time decay's rates and gaps in every slot) fit an SM, a tile's gap box
    starts on a 16-byte boundary, the tiles cover every time row once, and
    the workspace size covers the hand-off words."""
    B, T, D = shape
    W, R, S, cg, V = 6, 4, 2, 8, 4
    J = 32 // cg
    TC, TR = cg * V, W * J * R
    assert TR == 96 and TR % 4 == 0          # the gaps' box starts at ct TR: a 16-byte multiple
    n_dt, n_chunks = -(-D // TC), -(-T // TR)
    n_tiles = B * n_dt * n_chunks
    # the kernel's shared-memory layout: S slots (four operand boxes, then TC
    # rates and TR gaps), mbarriers, reader counts, warp and tile summaries,
    # incoming gradients, dL/dlambda sums and their warp count
    slot = -(-(4 * TR * TC * 4 + (TR + TC) * 4) // 128) * 128
    cnt = S * slot + S * 8
    tot = -(-(cnt + S * 4) // 16) * 16
    smem = tot + 2 * W * TC * 8 + 2 * TC * 8 + 2 * TC * 4 + 2 * TC * 4 + 16
    assert 2 * (smem + 1024) <= 228 * 1024          # two blocks per SM, 1 KB reserved each
    assert 2 * (W + 1) * 32 * 128 <= 65536          # at 128 registers per thread
    # processing rows of a tile: every time row of a chain exactly once
    rows = np.zeros(n_chunks * TR, dtype=np.int32)
    for ct in range(n_chunks):
        for w in range(W):
            for j in range(J):
                rho0 = (w * J + j) * R
                top = ct * TR + TR - 1 - rho0
                rows[top - R + 1:top + 1] += 1
    assert (rows == 1).all()
    lib = _abi.lib()
    kind = lib.sgr_backward_kernel(MINGRU, B, T, D, F32, 1)
    wide = B * n_dt * -(-T // 120) >= 2 * 148     # 15-warp blocks, 120-row tiles
    if n_tiles >= 4 * 148:                   # two tiles per block: the decayed gradient's plan
        assert lib.sgr_backward_workspace_size(MINGRU, B, T, D, F32) >= WS_HEADER + 8 * 3 * TC * n_tiles
    # the plain gradient (what the kernel query reports)
    assert kind == (2 if (n_tiles >= 4 * 148 and 2 * B * n_dt < 3 * 148) or wide else 1)
