"""ctypes view of the C ABI in include/pkv.h (argument marshalling only).

Loading builds ``libpkv.so`` in-tree first when it is missing or older than
its sources; any failure raises.  There is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

_lock = threading.Lock()
_lib = None

c_i32 = ctypes.c_int32
c_i64 = ctypes.c_int64
c_vp = ctypes.c_void_p
c_size = ctypes.c_size_t


class PkvPool(ctypes.Structure):
    _fields_ = [("k", c_vp), ("v", c_vp), ("num_layers", c_i64), ("num_slots", c_i64),
                ("layer_stride", c_i64), ("slot_stride", c_i64), ("num_kv_heads", c_i32),
                ("head_dim", c_i32), ("page_size", c_i32), ("dtype", c_i32),
                ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float)]


class PkvPageTable(ctypes.Structure):
    _fields_ = [("entries", c_vp), ("rows", c_i64), ("cols", c_i64), ("row_stride", c_i64)]


# Every symbol include/pkv.h declares, with its ctypes signature.
SIGNATURES = {
    "pkv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "pkv_version": (ctypes.c_char_p, []),
    "pkv_store_kv": (ctypes.c_int, [ctypes.POINTER(PkvPool), c_i32, c_vp, c_i64, c_vp, c_i64, c_vp,
                                    c_i32, c_i64, c_vp, c_vp]),
    "pkv_qk_norm_rope_store": (ctypes.c_int, [ctypes.POINTER(PkvPool), c_i32, c_vp, c_i64, c_i32, c_vp,
                                              c_i32, c_vp, c_i64, c_vp, c_vp, ctypes.c_float, c_vp,
                                              c_i32, c_i64, c_vp, c_vp, c_vp]),
    "pkv_selftest_wait_timeout": (ctypes.c_int, [c_vp, c_vp]),
    "pkv_workspace_create": (ctypes.c_int, [c_i32, c_i32, c_i64, ctypes.POINTER(c_vp)]),
    "pkv_workspace_destroy": (None, [c_vp]),
    "pkv_workspace_buffer": (c_vp, [c_vp, ctypes.POINTER(c_size)]),
    "pkv_workspace_error_word": (c_vp, [c_vp]),
    "pkv_read_device_error": (ctypes.c_int, [c_vp, c_vp, ctypes.POINTER(c_i32)]),
    "pkv_gather_kv": (ctypes.c_int, [ctypes.POINTER(PkvPool), c_i32, ctypes.POINTER(PkvPageTable),
                                     c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp]),
    "pkv_decode_workspace_bytes": (c_size, [c_i32, c_i32]),
    "pkv_decode_attn": (ctypes.c_int, [ctypes.POINTER(PkvPool), c_i32, c_vp, c_i32,
                                       ctypes.POINTER(PkvPageTable), c_vp, c_vp, c_i32,
                                       ctypes.c_float, c_vp, c_vp, c_size, c_vp, c_vp]),
    "pkv_decode_noalloc_max_scratch_bytes": (c_size, []),
    "pkv_decode_cascade_workspace_bytes": (c_size, [c_i32, c_i32, c_i64]),
    "pkv_decode_attn_cascade": (ctypes.c_int, [ctypes.POINTER(PkvPool), c_i32, c_vp, c_i32,
                                               ctypes.POINTER(PkvPageTable), c_vp, c_vp, c_i32,
                                               c_vp, c_vp, c_i32, c_i64, ctypes.c_float, c_vp,
                                               c_vp, c_size, c_vp, c_vp]),
    "pkv_decode_attn_noalloc": (ctypes.c_int, [ctypes.POINTER(PkvPool), c_i32, c_vp, c_i32,
                                               ctypes.POINTER(PkvPageTable), c_vp, c_vp, c_i32,
                                               ctypes.c_float, c_vp, c_vp, c_vp]),
    "pkv_extend_workspace_bytes": (c_size, [c_i32, c_i32, c_i64]),
    "pkv_extend_attn": (ctypes.c_int, [ctypes.POINTER(PkvPool), c_i32, c_vp, c_i32,
                                       ctypes.POINTER(PkvPageTable), c_vp, c_vp, c_vp, c_vp, c_i32,
                                       c_i64, c_i32, ctypes.c_float, c_vp, c_vp, c_size, c_vp,
                                       c_vp]),
}


def lib_path() -> str:
    return _build.LIB


def load() -> ctypes.CDLL:
    """Build if needed, then load libpkv.so and set argument types."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            lib = ctypes.CDLL(path, mode=ctypes.RTLD_GLOBAL)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
        return _lib


class PkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = load().pkv_status_string(status).decode()
        super().__init__(f"{where}: pkv status {status} ({msg})")
        self.status = status


def check(status: int, where: str) -> None:
    if status != 0:
        raise PkvError(status, where)
