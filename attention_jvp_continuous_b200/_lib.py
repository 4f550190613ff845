"""ctypes binding to ``libjvpattn.so`` (declared in include/jvp_attn.h).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels. The library is loaded on first use; a missing
library raises immediately (there is no fallback implementation).
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libjvpattn.so")

# Error codes (include/jvp_attn.h).
JVP_OK = 0
JVP_ERR_INVALID_ARG = -1
JVP_ERR_SHAPE_MISMATCH = -2
JVP_ERR_UNSUPPORTED_HEAD_DIM = -3
JVP_ERR_MISALIGNED = -4
JVP_ERR_LAUNCH_FAILED = -5
JVP_ERR_DEVICE_TIMEOUT = -6
JVP_ERR_DEVICE_BOUNDS = -7
JVP_ERR_OUT_OF_MEMORY = -8
JVP_ERR_UNSUPPORTED_DEVICE = -9
JVP_ERR_TOO_LARGE = -10

JVP_BF16 = 0
JVP_FP32 = 1

TILE_EMPTY, TILE_FULL, TILE_PARTIAL = 0, 1, 2

# Exported functions, as declared in include/jvp_attn.h.
EXPORTS = ("jvp_attn_fwd", "jvp_attn_fwd_noalloc", "jvp_attn_fwd_scatter", "jvp_attn_signal_barrier",
           "jvp_attn_bwd", "jvp_attn_bwd_scratch_len",
           "jvp_attn_cache_fwd", "jvp_attn_rope_copy", "jvp_attn_qkv_prologue",
           "jvp_attn_mask_stats",
           "jvp_attn_tile_classes", "jvp_attn_schedule", "jvp_attn_schedule_kv",
           "jvp_attn_check_device_error",
           "jvp_attn_set_wait_limit", "jvp_attn_set_stall_test", "jvp_attn_release", "jvp_attn_strerror",
           "jvp_attn_version")


class MaskDesc(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("tokens_per_frame", ctypes.c_int32),
                ("n_frames", ctypes.c_int32), ("chunk", ctypes.c_int32)]


class JvpAttnError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = code
        msg = strerror(code)
        super().__init__(f"{where}: {msg} ({code})" if where else f"{msg} ({code})")


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Load the library (once). Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"CUDA library {LIB_PATH} is missing; build it with "
                "`python -m attention_jvp_continuous_b200.build` "
                "(there is no non-CUDA implementation)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64p = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_int64)
        L.jvp_attn_fwd.argtypes = [vp] * 8 + [ctypes.POINTER(ctypes.c_float)] + \
            [i32] * 5 + [MaskDesc, ctypes.c_float, vp]
        L.jvp_attn_fwd.restype = i32
        L.jvp_attn_fwd_noalloc.argtypes = L.jvp_attn_fwd.argtypes
        L.jvp_attn_fwd_noalloc.restype = i32
        vpp = ctypes.POINTER(ctypes.c_void_p)
        L.jvp_attn_fwd_scatter.argtypes = [vp] * 6 + [vpp, vpp, vpp] + [i32] * 3 + \
            [i32] * 5 + [MaskDesc, ctypes.c_float, vp]
        L.jvp_attn_fwd_scatter.restype = i32
        L.jvp_attn_signal_barrier.argtypes = [vpp, i32, i32, ctypes.c_uint32, vp]
        L.jvp_attn_signal_barrier.restype = i32
        fp = ctypes.POINTER(ctypes.c_float)
        L.jvp_attn_bwd.argtypes = [vp] * 5 + [fp] + [vp] * 3 + [fp, ctypes.c_int64] + \
            [i32] * 5 + [MaskDesc, ctypes.c_float, vp]
        L.jvp_attn_bwd.restype = i32
        L.jvp_attn_bwd_scratch_len.argtypes = [i32, i32, i32]
        L.jvp_attn_bwd_scratch_len.restype = ctypes.c_int64
        L.jvp_attn_cache_fwd.argtypes = [vp] * 4 + [fp] + [i32] * 7 + [ctypes.c_float, vp]
        L.jvp_attn_cache_fwd.restype = i32
        L.jvp_attn_rope_copy.argtypes = [vp, vp] + [i32] * 9 + [fp, fp, i32, i32, vp]
        L.jvp_attn_rope_copy.restype = i32
        L.jvp_attn_qkv_prologue.argtypes = [vp] * 8 + [fp, fp, i32, ctypes.c_float, fp, fp] + \
            [i32] * 6 + [vp]
        L.jvp_attn_qkv_prologue.restype = i32
        L.jvp_attn_mask_stats.argtypes = [MaskDesc, i32, i32, i32, i64p, i64p, i64p, i64p]
        L.jvp_attn_mask_stats.restype = i32
        L.jvp_attn_tile_classes.argtypes = [MaskDesc, i32, i32, i32,
                                            ctypes.POINTER(ctypes.c_int8), ctypes.c_int64]
        L.jvp_attn_tile_classes.restype = i32
        i32p = ctypes.POINTER(ctypes.c_int32)
        L.jvp_attn_schedule.argtypes = [MaskDesc, i32, i32, i32, i32p, i32, i32p, i32,
                                        ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
        L.jvp_attn_schedule.restype = i32
        L.jvp_attn_schedule_kv.argtypes = L.jvp_attn_schedule.argtypes
        L.jvp_attn_schedule_kv.restype = i32
        L.jvp_attn_check_device_error.argtypes = [vp]
        L.jvp_attn_check_device_error.restype = i32
        L.jvp_attn_set_wait_limit.argtypes = [ctypes.c_uint64]
        L.jvp_attn_set_wait_limit.restype = i32
        L.jvp_attn_set_stall_test.argtypes = [i32]
        L.jvp_attn_set_stall_test.restype = i32
        L.jvp_attn_release.argtypes = []
        L.jvp_attn_release.restype = i32
        L.jvp_attn_strerror.argtypes = [i32]
        L.jvp_attn_strerror.restype = ctypes.c_char_p
        L.jvp_attn_version.argtypes = []
        L.jvp_attn_version.restype = i32
        _lib = L
        return L


def strerror(code: int) -> str:
    return lib().jvp_attn_strerror(int(code)).decode()


def check(code: int, where: str = "") -> None:
    if code != JVP_OK:
        raise JvpAttnError(code, where)
