"""ctypes loader for the in-tree CUDA library `_flce.so` (C ABI: include/flce.h).

Loading fails loudly: there is no CPU or PyTorch fallback for any FLCE step.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading


c_i32 = ctypes.c_int32
c_i64 = ctypes.c_int64
c_u64 = ctypes.c_uint64
c_f32 = ctypes.c_float
c_f64 = ctypes.c_double
c_size = ctypes.c_size_t
c_vp = ctypes.c_void_p

FLCE_OK = 0
STATUS_NAMES = {
    0: "FLCE_OK", 1: "FLCE_ERR_ARG", 2: "FLCE_ERR_SHAPE", 3: "FLCE_ERR_LABEL_RANGE",
    4: "FLCE_ERR_CUDA", 5: "FLCE_ERR_UNSUPPORTED", 6: "FLCE_ERR_TIMEOUT",
    7: "FLCE_ERR_WORKSPACE",
}
SUM, MEAN = 0, 1
BF16, FP32 = 0, 1
ACCUMULATE_DHIDDEN, ACCUMULATE_DWEIGHT = 1, 2
DHIDDEN_BF16, DWEIGHT_BF16 = 4, 8

# flce_option values (include/flce.h)
OPTIONS = {
    "cta_group": 0, "bwd_compact": 1, "bwd_fuse": 2, "mn3d": 3, "chunk_tokens": 4,
    "chunk_vocab": 5, "wait_timeout_ms": 6, "grad_tile_n": 7, "dz_tile_n": 8, "fwd_tile_n": 9,
    "fwd_group_m": 10, "dz_group_m": 11, "grad_group_m": 12, "fwd_dynamic": 13,
    "dz_buffers": 14, "fwd_compact": 15,
}

# Every symbol include/flce.h declares, with its ctypes signature.
SIGNATURES = {
    "flce_workspace_bytes": (c_size, [c_i64, c_i64, c_i64, c_i32]),
    "flce_workspace_bytes_ex": (c_size, [c_i64, c_i64, c_i64, c_i32, c_i32]),
    "flce_forward": (c_i32, [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_f32, c_i32,
                             c_i32, c_vp, c_vp, c_vp, c_vp, c_size, c_vp]),
    "flce_forward_ex": (c_i32, [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_f32, c_i32,
                                c_i32, c_f32, c_vp, c_vp, c_vp, c_vp, c_size, c_vp]),
    "flce_forward_ex2": (c_i32, [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_f32, c_i32,
                                 c_i32, c_f32, c_i64, c_vp, c_vp, c_vp, c_vp, c_size, c_vp]),
    "flce_backward": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_f32,
                              c_i32, c_i32, c_vp, c_f32, c_vp, c_vp, c_vp, c_i32, c_vp, c_size,
                              c_vp]),
    "flce_backward_ex": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_f32,
                                 c_i32, c_i32, c_vp, c_f32, c_i64, c_vp, c_vp, c_vp, c_i32, c_vp,
                                 c_size, c_vp]),
    "flce_set_option": (c_i32, [c_i32, c_i64]),
    "flce_get_option": (c_i32, [c_i32, ctypes.POINTER(c_i64)]),
    "flce_forward_noalloc": (c_i32, [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_f32,
                                     c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "flce_get_status": (c_i32, [c_vp, c_vp]),
    "flce_selftest_wait_timeout": (c_i32, [c_vp, c_i32, c_vp]),
    "flce_status_string": (ctypes.c_char_p, [c_i32]),
    "flce_version": (c_i32, []),
    "flce_launch_count": (c_u64, []),
    "flce_profile_enable": (c_i32, [c_i32]),
    "flce_profile_read": (c_i32, [c_i32, ctypes.POINTER(c_f64), ctypes.POINTER(c_i64)]),
}

_lib = None
_lock = threading.Lock()


class FlceError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


def library_path() -> str:
    from . import build as _build
    return _build.SO_PATH


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load (building first if needed) the CUDA library; raise if impossible."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        from . import build as _build
        path = library_path()
        if build_if_missing and _build.needs_build():
            _build.build()
        if not os.path.exists(path):
            raise RuntimeError(f"FLCE CUDA library not found at {path}; run "
                               "`python -m lm_head_linear_tmem_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def check(status: int, where: str) -> None:
    if status != FLCE_OK:
        raise FlceError(status, where)


def get_option(name: str) -> int:
    """Current value of a library option (see flce_option in include/flce.h)."""
    v = c_i64()
    check(load().flce_get_option(OPTIONS[name], ctypes.byref(v)), f"flce_get_option({name})")
    return int(v.value)


def set_option(name: str, value: int) -> None:
    """Set a process-wide library option (flce_set_option)."""
    check(load().flce_set_option(OPTIONS[name], int(value)), f"flce_set_option({name}={value})")


@contextlib.contextmanager
def options(**values):
    """Set library options for the duration of a `with` block, then restore them."""
    old = {k: get_option(k) for k in values}
    try:
        for k, v in values.items():
            set_option(k, v)
        yield
    finally:
        for k, v in old.items():
            set_option(k, v)
