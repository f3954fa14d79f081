"""ctypes view of ``libsgr.so`` (the C ABI in include/scan_gated_rnns.h).

Only declarations live here: names, argument and return types.  The library
is loaded on first use and a missing build raises immediately -- there is no
fallback implementation of any operation.
"""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsgr.so")

SGR_OK = 0
SGR_ERR_INVALID_ARG = 1
SGR_ERR_UNSUPPORTED = 2
SGR_ERR_WORKSPACE = 3
SGR_ERR_CUDA = 4
SGR_ERR_TIMEOUT = 5

SGR_F32 = 0
SGR_BF16 = 1

SGR_OP_MINGRU = 0
SGR_OP_MINMAX = 1
SGR_OP_MINGRU_LOG = 2

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t
_int = ctypes.c_int

SIGNATURES = {
    "mingru_scan": (_int, [_vp, _vp, _vp, _i64, _vp, _i64, _i64, _i64, _int, _vp, _sz, _vp]),
    "minmax_scan": (_int, [_vp, _vp, _vp, _i64, _vp, _i64, _i64, _i64, _int, _vp, _sz, _vp]),
    "mingru_scan_log": (_int, [_vp, _vp, _vp, _i64, _vp, _i64, _i64, _i64, _int, _vp, _sz, _vp]),
    "mingru_step": (_int, [_vp, _i64, _vp, _i64, _vp, _i64, _vp, _i64, _i64, _i64, _int, _vp]),
    "sgr_workspace_size": (_sz, [_int, _i64, _i64, _i64, _int]),
    "sgr_workspace_init": (_int, [_vp, _sz, _vp]),
    "sgr_workspace_status": (_int, [_vp, _sz, _int, _vp]),
    "sgr_status_string": (ctypes.c_char_p, [_int]),
    "sgr_version": (ctypes.c_char_p, []),
    "sgr_set_tile_override": (_int, [_int, _int]),
}



class Plan(ctypes.Structure):
    _fields_ = [("vector_path", ctypes.c_int32), ("kernel", ctypes.c_int32),
                ("channels_per_thread", ctypes.c_int32), ("channel_lanes", ctypes.c_int32),
                ("rows_per_thread", ctypes.c_int32), ("warps", ctypes.c_int32),
                ("threads", ctypes.c_int32), ("stages", ctypes.c_int32),
                ("tile_rows", ctypes.c_int64), ("tile_channels", ctypes.c_int64),
                ("n_channel_tiles", ctypes.c_int64), ("n_chains", ctypes.c_int64),
                ("n_chunks", ctypes.c_int64), ("n_tiles", ctypes.c_int64),
                ("smem_bytes", ctypes.c_uint64), ("workspace_bytes", ctypes.c_uint64),
                ("off_words", ctypes.c_uint64),
                ("div_chains_m", ctypes.c_uint32), ("div_chains_s", ctypes.c_uint32),
                ("div_dt_m", ctypes.c_uint32), ("div_dt_s", ctypes.c_uint32)]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


SIGNATURES.update({
    "sgr_scan_plan": (_int, [_int, _i64, _i64, _i64, _int, _int, ctypes.POINTER(Plan)]),
    "sgr_scan_plan_decay": (_int, [_i64, _i64, _i64, _int, _int, ctypes.POINTER(Plan)]),
    "sgr_set_wait_limit": (_int, [ctypes.c_uint32]),
    "sgr_set_drop_publish": (_int, [_i64]),
    "sgr_set_kernel_override": (_int, [_int]),
    "sgr_backward_kernel": (_int, [_int, _i64, _i64, _i64, _int, _int]),
    "mingru_scan_noalloc": (_int, [_vp, _vp, _vp, _i64, _vp, _i64, _i64, _i64, _int, _vp]),
    "sgr_host_staging_size": (_sz, [_int, _i64, _i64, _i64, _int, _int]),
    "mingru_scan_backward": (_int, [_vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _i64,
                                    _i64, _i64, _i64, _int, _vp, _sz, _vp]),
    "minmax_scan_backward": (_int, [_vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _i64,
                                    _i64, _i64, _i64, _int, _vp, _sz, _vp]),
    "sgr_backward_workspace_size": (_sz, [_int, _i64, _i64, _i64, _int]),
    "sgr_summary_workspace_size": (_sz, [_i64, _i64, _i64, _int]),
    "sgr_projected_workspace_size": (_sz, [_i64, _i64, _i64]),
    "mingru_projected_scan": (_int, [_vp, _vp, _vp, _i64, _vp, _i64, _i64, _i64, _i64, _vp, _sz, _vp]),
    "sgr_scan_summary": (_int, [_int, _vp, _vp, _i64, _i64, _i64, _int, _vp, _vp, _sz, _vp]),
    "sgr_combine_summaries": (_int, [_int, _vp, _i64, _vp, _i64, _vp, _i64, _i64, _i64, _int, _vp]),
    "mingru_scan_decay": (_int, [_vp, _vp, _vp, _i64, _vp, _i64, _vp, _int, _vp, _i64, _i64, _i64,
                                 _int, _vp, _sz, _vp]),
    "mingru_scan_decay_backward": (_int, [_vp, _vp, _vp, _i64, _vp, _i64, _vp, _int, _vp, _vp, _vp,
                                          _vp, _vp, _i64, _vp, _i64, _i64, _i64, _int, _vp, _sz,
                                          _vp]),
    "mingru_scan_host": (_int, [_vp, _vp, _vp, _i64, _vp, _i64, _i64, _i64, _int, _int, _vp, _sz, _vp]),
    "minmax_scan_host": (_int, [_vp, _vp, _vp, _i64, _vp, _i64, _i64, _i64, _int, _int, _vp, _sz, _vp]),
})

KERNEL_TILE = 1
KERNEL_PIPELINED = 2
KERNEL_PIPELINED_WIDE = 3
KERNEL_SEQUENTIAL = 4
KERNEL_SEQUENTIAL_SPLIT = 5
KERNEL_SEQUENTIAL_PAIR = 6
KERNEL_SEQUENTIAL_PAIR2 = 7
KERNEL_SEQUENTIAL_QUAD = 8

_lock = threading.Lock()
_lib = None


def lib():
    """The loaded library, with every entry point typed."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"{LIB_PATH} is missing: build it with "
                        "`python -m scan_gated_rnns_b200.build` (needs nvcc)")
                handle = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in SIGNATURES.items():
                    fn = getattr(handle, name)
                    fn.restype = res
                    fn.argtypes = args
                _lib = handle
    return _lib


def plan(op: int, B: int, T: int, D: int, dtype: int, aligned: bool = True, decay: bool = False) -> dict:
    """The library's plan for a scan of this shape; decay: the time-decayed
    minGRU's (op must then be SGR_OP_MINGRU)."""
    out = Plan()
    if decay:
        if op != SGR_OP_MINGRU:
            raise ValueError("plan: only the minGRU scan has a time-decayed form")
        check("sgr_scan_plan_decay", lib().sgr_scan_plan_decay(B, T, D, dtype, int(aligned), ctypes.byref(out)))
    else:
        check("sgr_scan_plan", lib().sgr_scan_plan(op, B, T, D, dtype, int(aligned), ctypes.byref(out)))
    return out.as_dict()


def status_string(code: int) -> str:
    return lib().sgr_status_string(code).decode()


class ScanError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {status_string(code)} (status {code})")


def check(fn: str, code: int) -> None:
    if code != SGR_OK:
        raise ScanError(fn, code)
