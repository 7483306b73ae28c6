"""ctypes declarations of the C ABI in ``include/fpstok.h`` (libfpstok.so).

The library is the in-tree ``libfpstok.so`` built by ``build.py``.  There is
no fallback: if the library is missing and cannot be built, loading raises.
"""
from __future__ import annotations

import ctypes
import os

from . import _build

P = ctypes.c_void_p
I = ctypes.c_int
I64 = ctypes.c_int64
SZ = ctypes.c_size_t

FPS_OK = 0
FPS_ERR_ARG = 1
FPS_ERR_TOO_LARGE = 2
FPS_ERR_WORKSPACE = 3
FPS_ERR_CUDA = 4
FPS_ERR_DEVICE = 5
FPS_ASSIGN_VORONOI = 0
FPS_ASSIGN_KNN = 1
FPS_MAX_K = 256
FPS_MAX_KNN = 128
FPS_MAX_F = 64

# (name, restype, argtypes) of every exported symbol, mirroring fpstok.h.
SIGNATURES = [
    ("fps_max_event_points", I64, []),
    ("fps_workspace_bytes", SZ, [I64, I, I, P]),
    ("fps_tokenize", I, [P, P, I, P, I, I64, P, P, P, P, P, P, P, P, P, SZ, P]),
    ("fps_host_workspace_bytes", SZ, [I64, I, I, P]),
    ("fps_tokenize_host", I, [P, P, I, P, I, I64, P, P, P, P, P, P, P, P, P, SZ, P]),
    ("fps_tokenize_static", I, [P, P, I, P, I, I64, P, P, P, P, P, P, P, P, P]),
    ("fps_static_device_status", I, [P, ctypes.POINTER(I)]),
    ("fps_assign_workspace_bytes", SZ, [I64, I]),
    ("fps_assign", I, [P, P, I, I64, P, P, I, P, P, P, SZ, P]),
    ("fps_knn_workspace_bytes", SZ, [I64, I]),
    ("fps_knn", I, [P, P, I, I64, P, P, I, I, P, P, P, SZ, P]),
    ("lloyd_workspace_bytes", SZ, [I64, I, I]),
    ("lloyd_refine", I, [P, P, I, I, P, I, I64, I, I, P, P, P, P, SZ, P]),
    ("segment_pool_workspace_bytes", SZ, [I64, I, I, I]),
    ("segment_pool", I, [P, I, P, I, I64, I, I, P, P, I, P, P, P, SZ, P]),
    ("segment_pool_backward_workspace_bytes", SZ, [I64, I, I, I, I]),
    ("segment_pool_backward", I, [P, I, P, I, I64, I, I, P, P, I, P, P, P, SZ, P]),
    ("fps_random_starts", I, [P, I, ctypes.c_uint64, ctypes.c_uint32, P, P]),
    ("fps_token_summaries_workspace_bytes", SZ, [I, I, I]),
    ("fps_token_summaries", I, [P, P, I, I, P, I, I64, I, P, P, P, P, P, SZ, P]),
    ("fps_pack_workspace_bytes", SZ, []),
    ("fps_pack_tokens", I, [P, I, P, P, I, I, P, P, P, P, SZ, P]),
    ("fps_unpack_tokens", I, [P, I, I64, P, I, I, P, P, SZ, P]),
    ("fps_device_status", I, [P, P, ctypes.POINTER(I)]),
    ("fps_status_string", ctypes.c_char_p, [I]),
    ("fps_launch_count", ctypes.c_uint64, []),
    ("fps_set_exchange_test", None, [I, I]),
    ("fps_set_stage_events", None, [ctypes.POINTER(P), I]),
    ("fps_stage_mask", ctypes.c_uint, []),
    ("fps_schedule_for", I, [I64, I, I]),
]


class FpsOpts(ctypes.Structure):
    """``fps_opts`` of fpstok.h."""

    _fields_ = [("K", I), ("assign_mode", I), ("k", I), ("lloyd_iters", I), ("charge_col", I),
                ("force_schedule", I), ("max_event_hint", I), ("axis_scale", ctypes.c_float * 4)]


_lib = None


def library_path() -> str:
    return _build.LIB


def load(build_if_missing: bool = True):
    """Load (building first if needed) libfpstok.so and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.LIB
    if build_if_missing and (not os.path.exists(path) or _build.stale()):
        _build.build()
    if not os.path.exists(path):
        raise RuntimeError(f"fpstok CUDA library not found at {path}; run build()")
    lib = ctypes.CDLL(path)
    for name, res, args in SIGNATURES:
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class FpsError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = load().fps_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


def check(status: int, where: str) -> None:
    if status != FPS_OK:
        raise FpsError(status, where)
