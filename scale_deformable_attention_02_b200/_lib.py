"""ctypes view of libmsda.so (the C ABI in include/msda.h, include/msda_tiled.h
and include/msda_debug.h) and of its bounds-checked build libmsda_checked.so
(plus include/msda_checked.h).  No fallback: if a library is missing or does
not load, every call raises."""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmsda.so")
LIB_CHECKED_PATH = os.path.join(PKG, "libmsda_checked.so")

MSDA_F32 = 0
MSDA_BF16 = 1

STATUS_NAMES = {
    0: "MSDA_OK", 1: "MSDA_ERR_NULL", 2: "MSDA_ERR_SHAPE", 3: "MSDA_ERR_LEVELS",
    4: "MSDA_ERR_DTYPE", 5: "MSDA_ERR_ALIGN", 6: "MSDA_ERR_ALIAS",
    7: "MSDA_ERR_UNSUPPORTED", 8: "MSDA_ERR_CUDA", 9: "MSDA_ERR_DEVICE_CHECK",
}

# Every function declared in include/*.h, with its ctypes signature.
P = ctypes.c_void_p
I64 = ctypes.c_int64
INT = ctypes.c_int


class Dims(ctypes.Structure):
    _fields_ = [(k, ctypes.c_int64) for k in ("N", "Lq", "S", "M", "D", "L", "K")]


TILE_MAX_LEVELS = 8
I32 = ctypes.c_int32


class TilePlan(ctypes.Structure):
    """msda_tile_plan (include/msda_tiled.h)."""
    _fields_ = [("N", ctypes.c_int64), ("Lq", ctypes.c_int64), ("S", ctypes.c_int64),
                ("L", ctypes.c_int64), ("D", ctypes.c_int64), ("value_dtype", I32),
                ("halo", I32), ("grid_x", I32), ("grid_y", I32), ("ctas_per_sm", I32),
                ("reserved", I32), ("shapes", ctypes.c_int64 * (2 * TILE_MAX_LEVELS)),
                ("window_w", I32 * TILE_MAX_LEVELS), ("window_h", I32 * TILE_MAX_LEVELS),
                ("window_bytes", ctypes.c_int64), ("device_bytes", ctypes.c_int64)]


SIGNATURES = {
    "msda_status_string": (ctypes.c_char_p, [INT]),
    "msda_abi_version": (INT, []),
    "msda_last_cuda_error": (INT, []),
    "msda_level_start_index": (INT, [P, I64, P, P]),
    "msda_forward": (INT, [P, INT, P, P, P, P, P, Dims, P]),
    "msda_forward_fused": (INT, [P, INT, P, P, P, INT, P, P, P, P, P, Dims, P]),
    "msda_backward": (INT, [P, INT, P, P, P, P, P, P, P, P, Dims, P]),
    "msda_backward_fused": (INT, [P, INT, P, P, P, INT, P, P, P, P, P, P, P, Dims, P]),
    "msda_forward_grouped": (INT, [P, INT, P, P, P, P, P, Dims, I64, P]),
    "msda_forward_fused_grouped": (INT, [P, INT, P, P, P, INT, P, P, P, P, P, Dims, I64, P]),
    "msda_backward_grouped": (INT, [P, INT, P, P, P, P, P, P, P, P, Dims, I64, P]),
    "msda_backward_fused_grouped": (INT, [P, INT, P, P, P, INT, P, P, P, P, P, P, P, Dims, I64,
                                          P]),
    "msda_tile_plan_init": (INT, [INT, P, P, Dims, INT, INT, P]),
    "msda_tile_plan_build": (INT, [P, P, INT, P, P]),
    "msda_forward_tiled": (INT, [P, INT, P, P, P, P, P, Dims, P, P, P]),
    "msda_forward_fused_tiled": (INT, [P, INT, P, P, P, INT, P, P, P, P, P, Dims, P, P, P]),
    "msda_backward_tiled": (INT, [P, INT, P, P, P, P, P, P, P, P, Dims, P, P, P]),
    "msda_forward_fused_tiled_noalloc": (INT, [P, INT, P, P, P, INT, P, P, P, P, P, Dims, INT,
                                               INT, P]),
    "msda_backward_fused_tiled": (INT, [P, INT, P, P, P, INT, P, P, P, P, P, P, P, Dims, P, P,
                                        P]),
    "msda_debug_sample_points": (INT, [P, P, P, Dims, P, P, P, P, P, P, P]),
    "msda_debug_row_traffic": (INT, [INT, P, INT, P, I64, P, I64, P, I64, INT, INT, P]),
    "msda_debug_tiled_stalls": (INT, [P]),
}

# Only in libmsda_checked.so (include/msda_checked.h).
CHECKED_SIGNATURES = {
    "msda_checked_set_limit": (INT, [I64]),
    "msda_checked_last_violation": (INT, [P, P]),
}

_lock = threading.Lock()
_libs: dict = {}
_route = threading.local()  # .checked: this thread's binding calls use the checked build


def _open(path: str, signatures: dict) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is not built; run `python -m "
            "scale_deformable_attention_02_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in signatures.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load(checked: bool | None = None) -> ctypes.CDLL:
    """Load libmsda.so, or libmsda_checked.so when `checked` is true (None: the
    library the calling thread routes to, see api.checked_library)."""
    if checked is None:
        checked = getattr(_route, "checked", False)
    with _lock:
        if checked not in _libs:
            if checked:
                _libs[True] = _open(LIB_CHECKED_PATH, {**SIGNATURES, **CHECKED_SIGNATURES})
            else:
                _libs[False] = _open(LIB_PATH, SIGNATURES)
        return _libs[checked]


def status_string(code: int) -> str:
    return load().msda_status_string(int(code)).decode()
