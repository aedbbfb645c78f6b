"""ctypes binding of include/kv.h: the same entry points, argument marshalling only.

Every function here forwards to `libpkv.so`; all paging, planning and
attention happens in the library. Loading fails loudly if the library has not
been built (there is no fallback).
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libpkv.so")

KV_OK = 0
KV_ERR_ARG = -1
KV_ERR_CAPACITY = -2
KV_ERR_ORDER = -3
KV_ERR_NO_PENDING = -4
KV_ERR_NOT_APPENDED = -5
KV_ERR_EMPTY = -6
KV_ERR_CUDA = -7
KV_ERR_DEVICE_CHECK = -8
KV_ERR_UNSUPPORTED = -9
KV_ERR_STALE_PLAN = -10
KV_BF16 = 0
KV_FP16 = 1
KV_MAX_STREAMS = 32
KV_STATIC_SCRATCH_BYTES = 32 << 20
KV_NOT_CURRENT = -0x40000000   # krow of a tile that is not the open step's frame

ERR_NAMES = {
    KV_ERR_ARG: "ARG", KV_ERR_CAPACITY: "CAPACITY", KV_ERR_ORDER: "ORDER",
    KV_ERR_NO_PENDING: "NO_PENDING", KV_ERR_NOT_APPENDED: "NOT_APPENDED", KV_ERR_EMPTY: "EMPTY",
    KV_ERR_CUDA: "CUDA", KV_ERR_DEVICE_CHECK: "DEVICE_CHECK", KV_ERR_UNSUPPORTED: "UNSUPPORTED",
    KV_ERR_STALE_PLAN: "STALE_PLAN",
}


class kv_stats(ctypes.Structure):
    _fields_ = [("frame_count", ctypes.c_int), ("scale_pages", ctypes.c_int),
                ("live_pages", ctypes.c_int), ("free_pages", ctypes.c_int),
                ("special_tokens", ctypes.c_int)]


class kv_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "max_pages", "page_size", "num_heads", "head_dim", "scale_frames", "window", "num_blocks",
        "num_special", "dtype", "patch_pages", "special_base", "special_pages", "tokens_per_frame",
        "cross_frame_special", "camera_only")]


class kv_plan_stats(ctypes.Structure):
    _fields_ = [("n_streams", ctypes.c_int), ("n_ctas", ctypes.c_int),
                ("n_split_units", ctypes.c_int), ("n_kv_tiles", ctypes.c_int),
                ("tiles_per_cta", ctypes.c_int), ("visible_tokens", ctypes.c_longlong),
                ("fused_merge", ctypes.c_int), ("run_launches", ctypes.c_int),
                ("upload_launches", ctypes.c_int)]


class KVError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str):
        self.code = code
        self.name = ERR_NAMES.get(code, str(code))
        super().__init__(f"{where}: KV_ERR_{self.name} ({detail})")


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_IP = ctypes.POINTER(ctypes.c_int)

# name -> (restype, argtypes)
SIGNATURES = {
    "kv_init": (_I, [ctypes.POINTER(_P), _I, _I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "kv_init_group": (_I, [ctypes.POINTER(_P), _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "kv_destroy": (None, [_P]),
    "kv_reset": (_I, [_P]),
    "kv_pool_bytes": (_SZ, [_P]),
    "kv_bind_pool": (_I, [_P, _I, _P, _P]),
    "kv_append_frame": (_I, [_P, _I, _P, _P, _P]),
    "kv_evict_frames": (_I, [_P]),
    "kv_defer_eviction": (_I, [_P, _I]),
    "kv_commit_frame": (_I, [_P]),
    "kv_rollback_last_frame": (_I, [_P]),
    "kv_get_stats": (_I, [_P, ctypes.POINTER(kv_stats)]),
    "kv_get_free_list": (_I, [_P, _IP, _I, _IP]),
    "kv_get_config": (_I, [_P, ctypes.POINTER(kv_config)]),
    "kv_workspace_bytes": (_SZ, [ctypes.POINTER(_P), _I]),
    "kv_plan": (_I, [ctypes.POINTER(_P), ctypes.POINTER(_P), _I, _I, _P, _SZ, _P]),
    "kv_run": (_I, [_P, _I, _P, _P, _P]),
    "kv_run_append": (_I, [_P, _I, _P, _P, _P, _P, _P]),
    "kv_begin_frame": (_I, [_P]),
    "kv_plan_free": (None, [_P]),
    "kv_get_page_table": (_I, [_P, _I, _IP, _I, _IP, _IP]),
    "kv_get_kv_tiles": (_I, [_P, _I, _IP, _IP, _IP, _IP, _IP, _I, _IP]),
    "kv_plan_get_stats": (_I, [_P, ctypes.POINTER(kv_plan_stats)]),
    "kv_check_device": (_I, [_P, _P]),
    "kv_run_static": (_I, [ctypes.POINTER(_P), _I, _I, _I, _P, _P, _I, _P]),
    "kv_set_cross_frame_special": (_I, [_P, _I]),
    "kv_set_camera_only": (_I, [_P, _I]),
    "kv_testing_fail_launches": (None, [_I]),
    "kv_strerror": (ctypes.c_char_p, [_I]),
    "kv_last_error": (ctypes.c_char_p, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (RTLD_GLOBAL not needed). Raises if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_frame_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def check(rc: int, where: str) -> None:
    if rc != KV_OK:
        raise KVError(rc, where, lib().kv_last_error().decode())


def strerror(rc: int) -> str:
    return lib().kv_strerror(rc).decode()
