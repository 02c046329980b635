"""ctypes declarations of the C ABI in include/svt.h (libsvt.so).

Loading fails loudly when the library has not been built: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsvt.so")

SVT_OK, SVT_EINVAL, SVT_ENOPAGES, SVT_ESTATE, SVT_ECUDA, SVT_EDEVICE = 0, -1, -2, -3, -4, -5
STATUS_NAMES = {0: "SVT_OK", -1: "SVT_EINVAL", -2: "SVT_ENOPAGES", -3: "SVT_ESTATE",
                -4: "SVT_ECUDA", -5: "SVT_EDEVICE"}
SVT_BF16, SVT_FP16, SVT_FP32 = 0, 1, 2
MAX_STREAMS = 32

EXPORTED = [
    "svt_default_opts", "svt_pool_bytes", "svt_create_cache", "svt_destroy_cache", "svt_reset",
    "svt_set_free_lists", "svt_append_frame", "svt_evict_frames", "svt_set_defer_eviction",
    "svt_execute_deferred_eviction", "svt_rollback_last_frame", "svt_build_visible_page_table",
    "svt_get_page_table", "svt_read_device_page_table", "svt_plan", "svt_plan_extra",
    "svt_get_plan_info", "svt_run", "svt_run_extra", "svt_frame_step", "svt_get_graph_counts", "svt_get_cache_stats",
    "svt_device_error", "svt_last_error",
    "svt_attention_noalloc", "svt_noalloc_device_error", "svt_selftest_wait_limit",
]


class CacheOpts(ctypes.Structure):
    _fields_ = [
        ("num_blocks", ctypes.c_int), ("num_special", ctypes.c_int),
        ("num_streams", ctypes.c_int), ("dtype", ctypes.c_int),
        ("patch_pages", ctypes.c_int), ("max_qo_len", ctypes.c_int),
        ("max_splits", ctypes.c_int), ("rope_grid", ctypes.c_int),
        ("rope_theta", ctypes.c_float), ("host_only", ctypes.c_int),
        ("pool", ctypes.c_void_p), ("no_cross_frame_special", ctypes.c_int),
    ]


class Stats(ctypes.Structure):
    _fields_ = [("frame_count", ctypes.c_int64), ("scale_pages", ctypes.c_int64),
                ("live_pages", ctypes.c_int64), ("free_pages", ctypes.c_int64),
                ("special_tokens", ctypes.c_int64)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("num_items", ctypes.c_int),
                ("splits", ctypes.c_int * MAX_STREAMS),
                ("kv_tiles", ctypes.c_int * MAX_STREAMS),
                ("kv_tokens", ctypes.c_int64 * MAX_STREAMS),
                ("qo_len", ctypes.c_int64 * MAX_STREAMS)]


_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m streaming_video_transformer_b200.build`"
            " (there is no fallback path)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, VP = ctypes.POINTER, ctypes.c_int, ctypes.c_void_p
    i32p = P(ctypes.c_int32)
    sig = {
        "svt_default_opts": (None, [P(CacheOpts)]),
        "svt_pool_bytes": (ctypes.c_size_t, [I, I, I, I, P(CacheOpts)]),
        "svt_create_cache": (I, [I, I, I, I, I, I, P(CacheOpts), P(VP)]),
        "svt_destroy_cache": (I, [VP]),
        "svt_reset": (I, [VP]),
        "svt_set_free_lists": (I, [VP, i32p, I, i32p, I]),
        "svt_append_frame": (I, [VP, I, I, VP, VP, VP]),
        "svt_evict_frames": (I, [VP, I]),
        "svt_set_defer_eviction": (I, [VP, I, I]),
        "svt_execute_deferred_eviction": (I, [VP, I]),
        "svt_rollback_last_frame": (I, [VP, I]),
        "svt_build_visible_page_table": (I, [VP, VP]),
        "svt_get_page_table": (I, [VP, i32p, i32p, i32p, I, P(I)]),
        "svt_read_device_page_table": (I, [VP, i32p, i32p, i32p, I, P(I), VP]),
        "svt_plan": (I, [VP, i32p, VP]),
        "svt_plan_extra": (I, [VP, i32p, i32p, VP]),
        "svt_get_plan_info": (I, [VP, P(PlanInfo)]),
        "svt_run": (I, [VP, I, VP, VP, VP, I, VP]),
        "svt_run_extra": (I, [VP, I, VP, VP, VP, VP, VP, I, VP]),
        "svt_frame_step": (I, [VP, I, P(VP), P(VP), P(VP), P(VP), I, VP]),
        "svt_get_graph_counts": (I, [VP, P(I), P(I)]),
        "svt_get_cache_stats": (I, [VP, I, P(Stats)]),
        "svt_device_error": (I, [VP, VP]),
        "svt_last_error": (ctypes.c_char_p, []),
        "svt_attention_noalloc": (I, [VP, VP, VP, VP, VP, i32p, i32p, i32p, I, I, I, I, I, I, I,
                                      VP]),
        "svt_noalloc_device_error": (I, [VP]),
        "svt_selftest_wait_limit": (I, [I, VP]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib
