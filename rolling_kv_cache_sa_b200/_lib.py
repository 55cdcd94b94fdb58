"""ctypes declarations of libsa.so (include/sa.h). Argument marshalling only."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# SA_LIBRARY_VARIANT=debug loads the debug build (index checks in every kernel,
# sa_debug_bounds_status); anything else the normal build
LIB_PATH = os.path.join(_HERE, "libsa_debug.so" if os.environ.get("SA_LIBRARY_VARIANT") == "debug"
                        else "libsa.so")

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_OOM, SA_ERR_CUDA, SA_ERR_STATE, \
    SA_ERR_DEVICE_TIMEOUT, SA_ERR_DEVICE_BOUNDS = range(8)
STATUS_NAMES = {0: "SA_OK", 1: "SA_ERR_INVALID_ARG", 2: "SA_ERR_UNSUPPORTED", 3: "SA_ERR_OOM",
                4: "SA_ERR_CUDA", 5: "SA_ERR_STATE", 6: "SA_ERR_DEVICE_TIMEOUT",
                7: "SA_ERR_DEVICE_BOUNDS"}
SA_F32, SA_BF16, SA_BF16_E4M3 = 0, 1, 2
SA_SINK_SHIFT, SA_SINK_REPIN = 0, 1
SA_MAX_CHUNK_FRAMES = 32

# every symbol include/sa.h declares
EXPORTED = (
    "sa_cache_create", "sa_append_attend", "sa_rope_refresh", "sa_cache_reset",
    "sa_cache_destroy", "sa_append_attend_host", "sa_stream_state", "sa_cache_copy_out",
    "sa_get_device_status", "sa_plan_chunk", "sa_refresh_delta", "sa_profile_begin",
    "sa_profile_end", "sa_last_error_string", "sa_abi_version", "sa_append_attend_noalloc",
    "sa_profile_launches", "sa_wait_probe", "sa_attend", "sa_cache_set_sink_mode",
    "sa_sink_update", "sa_append_attend_host_async", "sa_host_wait", "sa_cache_set_fp8_scales",
    "sa_cache_export_size", "sa_cache_export", "sa_cache_import", "sa_cache_get_fp8_scales",
    "sa_gdn_chunk", "sa_gdn_workspace_size", "sa_noalloc_device_status",
    "sa_debug_bounds_status", "sa_debug_bounds_selftest", "sa_gdn_device_status",
)


class sa_config(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("frame_h", ctypes.c_int32), ("frame_w", ctypes.c_int32),
        ("chunk_frames", ctypes.c_int32), ("sink_frames", ctypes.c_int32),
        ("window_frames", ctypes.c_int32), ("rope_dims", ctypes.c_int32 * 3),
        ("rope_base", ctypes.c_float), ("softmax_scale", ctypes.c_float),
        ("dtype", ctypes.c_int32),
    ]


class sa_gdn_config(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("tokens", ctypes.c_int64), ("scale", ctypes.c_float),
        ("pad_", ctypes.c_int32),
    ]


class sa_chunk_plan(ctypes.Structure):
    _fields_ = [
        ("chunk", ctypes.c_int64), ("sink_len", ctypes.c_int64), ("ring_len", ctypes.c_int64),
        ("n_keys", ctypes.c_int64), ("n_frames", ctypes.c_int32), ("pad_", ctypes.c_int32),
        ("dest_row", ctypes.c_int64 * SA_MAX_CHUNK_FRAMES),
        ("t_pos", ctypes.c_int64 * SA_MAX_CHUNK_FRAMES),
        ("is_sink", ctypes.c_int32 * SA_MAX_CHUNK_FRAMES),
    ]


class SAError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_LIB = None


def lib() -> ctypes.CDLL:
    """Loads libsa.so; raises if it is missing (there is no fallback path)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: the CUDA library must be built "
                           "(__graft_entry__.build()); there is no fallback path")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    P = ctypes.POINTER
    sig = {
        "sa_cache_create": [P(sa_config), vp, P(vp)],
        "sa_append_attend": [vp, vp, vp, vp, vp, vp, vp],
        "sa_attend": [vp, vp, vp, vp, vp, vp, vp],
        "sa_cache_set_sink_mode": [vp, i32],
        "sa_cache_set_fp8_scales": [vp, vp, vp, vp],
        "sa_cache_get_fp8_scales": [vp, vp, vp, vp],
        "sa_cache_export_size": [vp, P(ctypes.c_size_t)],
        "sa_cache_export": [vp, vp, ctypes.c_size_t, vp],
        "sa_cache_import": [vp, vp, ctypes.c_size_t, vp],
        "sa_sink_update": [vp, vp, vp, ctypes.c_float, vp, vp],
        "sa_rope_refresh": [vp, vp, vp],
        "sa_cache_reset": [vp, vp],
        "sa_cache_destroy": [vp],
        "sa_append_attend_host": [vp, vp, vp, vp, vp, vp, vp],
        "sa_append_attend_host_async": [vp, vp, vp, vp, vp, vp, vp],
        "sa_host_wait": [vp],
        "sa_stream_state": [vp, i32, P(i64), P(i64)],
        "sa_cache_copy_out": [vp, i32, vp, vp, vp],
        "sa_get_device_status": [vp, vp],
        "sa_plan_chunk": [P(sa_config), i64, i64, P(sa_chunk_plan)],
        "sa_refresh_delta": [P(sa_config), i64, i64, P(i64)],
        "sa_profile_begin": [vp],
        "sa_profile_launches": [vp, P(i64)],
        "sa_wait_probe": [ctypes.c_uint64, P(i64), vp],
        "sa_append_attend_noalloc": [P(sa_config), vp, vp, vp, P(i64), P(i64), vp, vp, vp, vp,
                                     vp, vp],
        "sa_gdn_chunk": [P(sa_gdn_config), vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp,
                         vp],
        "sa_gdn_workspace_size": [P(sa_gdn_config), P(ctypes.c_size_t)],
        "sa_noalloc_device_status": [vp],
        "sa_debug_bounds_status": [vp],
        "sa_debug_bounds_selftest": [vp],
        "sa_gdn_device_status": [vp, vp],
        "sa_profile_end": [vp, P(ctypes.c_double), P(i32), P(ctypes.c_double), P(i32),
                           P(ctypes.c_double), P(i32)],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.sa_last_error_string.argtypes = []
    L.sa_last_error_string.restype = ctypes.c_char_p
    L.sa_abi_version.argtypes = []
    L.sa_abi_version.restype = ctypes.c_int32
    _LIB = L
    return L


def check(status: int, where: str) -> None:
    if status != SA_OK:
        raise SAError(status, where, lib().sa_last_error_string().decode())
