"""ctypes declarations of librf2.so (the C ABI in include/rf2.h).  Argument marshalling only."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librf2.so")

RF2_OK = 0
RF2_ERR_INVALID_ARG = 1
RF2_ERR_UNSUPPORTED = 2
RF2_ERR_ALIGNMENT = 3
RF2_ERR_WORKSPACE = 4
RF2_ERR_BAD_INDEX = 5
RF2_ERR_TIMEOUT = 6
RF2_ERR_CUDA = 7

RF2_SINK_ADDITIVE = 1
RF2_CHECKED = 2
RF2_RASTER = 4
RF2_NO_PERMUTE = 8
RF2_FP8 = 16
RF2_NOALLOC_SCRATCH_BYTES = 16 << 20

# Every symbol include/rf2.h declares.
EXPORTS = (
    "rf2_permute",
    "rf2_unpermute",
    "rf2_kept_count",
    "rf2_workspace_size",
    "rf2_predict_mask",
    "rf2_predict_mask_noalloc",
    "rf2_sparse_attn",
    "rf2_attention",
    "rf2_schedule_action",
    "rf2_quantize_fp8",
    "rf2_sparse_attn_fp8",
    "rf2_v1_kmax",
    "rf2_v1_workspace_size",
    "rf2_v1_predict_mask",
    "rf2_selftest_wait_timeout",
    "rf2_status_string",
)

RF2_V1_TEMPORAL = 0
RF2_V1_SPATIAL = 1
RF2_V1_TEXTURAL = 2


RF2_STEP_DENSE = 0
RF2_STEP_PREDICT = 1
RF2_STEP_REUSE = 2


class Rf2Schedule(ctypes.Structure):
    _fields_ = [("total_steps", ctypes.c_int), ("dense_fraction", ctypes.c_double),
                ("predict_interval", ctypes.c_int)]


class Rf2V1Params(ctypes.Structure):
    _fields_ = [("bandwidth", ctypes.c_double), ("tau", ctypes.c_int), ("alpha", ctypes.c_double),
                ("omega", ctypes.c_int), ("dynamic", ctypes.c_int), ("recall_target", ctypes.c_double)]


class Rf2Geom(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "heads", "T", "H", "W", "D", "wt", "wh", "ww")]


_vp = ctypes.c_void_p
_i32p = ctypes.c_void_p  # device int32* passed as a raw address
_gp = ctypes.POINTER(Rf2Geom)

_SIGS = {
    "rf2_permute": (ctypes.c_int, [_vp, _vp, _gp, _vp]),
    "rf2_unpermute": (ctypes.c_int, [_vp, _vp, _gp, _vp]),
    "rf2_kept_count": (ctypes.c_int, [_gp, ctypes.c_double, ctypes.c_int, ctypes.c_uint]),
    "rf2_workspace_size": (ctypes.c_size_t, [_gp, ctypes.c_double, ctypes.c_int, ctypes.c_uint,
                                             ctypes.c_int]),
    "rf2_predict_mask": (ctypes.c_int, [_vp, _vp, _gp, ctypes.c_double, ctypes.c_int, ctypes.c_uint,
                                        _i32p, _i32p, ctypes.c_int, _vp, ctypes.c_size_t, _vp]),
    "rf2_predict_mask_noalloc": (ctypes.c_int, [_vp, _vp, _gp, ctypes.c_double, ctypes.c_int,
                                                ctypes.c_uint, _i32p, _i32p, ctypes.c_int, _vp]),
    "rf2_sparse_attn": (ctypes.c_int, [_vp, _vp, _vp, _i32p, _i32p, ctypes.c_int, _gp, ctypes.c_float,
                                       _vp, _i32p, ctypes.c_uint, _vp]),
    "rf2_attention": (ctypes.c_int, [_vp, _vp, _vp, _gp, ctypes.c_double, ctypes.c_int, ctypes.c_float,
                                     _vp, _i32p, _vp, ctypes.c_size_t, ctypes.c_uint, _vp]),
    "rf2_schedule_action": (ctypes.c_int, [ctypes.POINTER(Rf2Schedule), ctypes.c_int]),
    "rf2_quantize_fp8": (ctypes.c_int, [_vp, _vp, _vp, _gp, ctypes.c_uint, _vp, _vp, _vp, _vp, _vp]),
    "rf2_sparse_attn_fp8": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32p, _i32p, ctypes.c_int, _gp, ctypes.c_float,
                                           _vp, _i32p, ctypes.c_uint, _vp]),
    "rf2_v1_kmax": (ctypes.c_int, [_gp, ctypes.POINTER(Rf2V1Params), ctypes.c_uint]),
    "rf2_v1_workspace_size": (ctypes.c_size_t, [_gp, ctypes.POINTER(Rf2V1Params), ctypes.c_uint]),
    "rf2_v1_predict_mask": (ctypes.c_int, [_vp, _vp, _gp, ctypes.POINTER(Rf2V1Params), ctypes.c_uint, _i32p,
                                           _i32p, ctypes.c_int, _i32p, _vp, _vp, ctypes.c_size_t, _vp]),
    "rf2_selftest_wait_timeout": (ctypes.c_int, [_i32p, ctypes.c_double, ctypes.c_double, _vp]),
    "rf2_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load librf2.so (once).  Raises if it has not been built: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(
                f"librf2.so not found at {path}; build it with "
                "`python -m image_diffusion_dits_b200.build` (needs nvcc)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib
