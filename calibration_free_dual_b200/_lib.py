"""ctypes declarations of libdq.so (the C ABI in include/dq.h); marshalling only."""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdq.so")

c_void_p, c_int32, c_int64, c_size_t = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t

DQ_OK, DQ_ERR_INVALID_ARG, DQ_ERR_SHAPE, DQ_ERR_DTYPE, DQ_ERR_WORKSPACE = 0, 1, 2, 3, 4
DQ_ERR_NONFINITE, DQ_ERR_TIMEOUT, DQ_ERR_CUDA, DQ_ERR_UNSUPPORTED = 5, 6, 7, 8
DQ_INT4, DQ_MXINT4, DQ_MXFP4, DQ_NVFP4, DQ_INT8, DQ_MXINT8 = 0, 1, 2, 3, 4, 5
DQ_F32, DQ_BF16 = 0, 1
DQ_CODEC_INT4, DQ_CODEC_E2M1, DQ_CODEC_E4M3, DQ_CODEC_E8M0, DQ_CODEC_BF16 = 0, 1, 2, 3, 4
DQ_CODEC_INT8 = 5
DQ_NOALLOC_SCRATCH_BYTES = 4 << 20
DQ_UPDATE_BOTH, DQ_UPDATE_ROW_ONLY, DQ_UPDATE_COL_ONLY = 0, 1, 2


class dq_format(ctypes.Structure):
    _fields_ = [("kind", c_int32), ("group", c_int32)]


class dq_matrix(ctypes.Structure):
    _fields_ = [("W", c_void_p), ("m", c_int64), ("n", c_int64), ("ldw", c_int64),
                ("r0", c_void_p), ("c0", c_void_p), ("q_packed", c_void_p), ("r", c_void_p),
                ("c", c_void_p), ("block_scales", c_void_p), ("tensor_scale", c_void_p),
                ("mse_trace", c_void_p)]


class dq_solve_options(ctypes.Structure):
    _fields_ = [("update", c_int32), ("qchange", ctypes.POINTER(c_void_p))]


# name -> (restype, argtypes); the same names as the C ABI
SIGNATURES = {
    "dq_status_string": (ctypes.c_char_p, [c_int32]),
    "dq_solve_max_rows": (c_int64, [c_int64, dq_format, c_int32]),
    "dq_solve_workspace_bytes": (c_size_t, [c_int64, ctypes.POINTER(c_int64),
                                            ctypes.POINTER(c_int64), dq_format, c_int32]),
    "dq_solve_batched": (c_int32, [ctypes.POINTER(dq_matrix), c_int64, c_int32, dq_format,
                                   c_int32, c_void_p, c_size_t, c_void_p]),
    "dq_solve_workspace_bytes_ex": (c_size_t, [c_int64, ctypes.POINTER(c_int64),
                                               ctypes.POINTER(c_int64), dq_format, c_int32,
                                               ctypes.POINTER(dq_solve_options)]),
    "dq_solve_batched_ex": (c_int32, [ctypes.POINTER(dq_matrix), c_int64, c_int32, dq_format,
                                      c_int32, ctypes.POINTER(dq_solve_options), c_void_p,
                                      c_size_t, c_void_p]),
    "dq_solve": (c_int32, [c_void_p, c_int32, c_int64, c_int64, c_int64, dq_format, c_int32,
                           c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                           c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "dq_solve_noalloc": (c_int32, [c_void_p, c_int32, c_int64, c_int64, c_int64, dq_format,
                                   c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                   c_void_p, c_void_p, c_void_p, c_void_p]),
    "dq_act_quant_workspace_bytes": (c_size_t, [c_int64, c_int64, dq_format]),
    "dq_act_quant": (c_int32, [c_void_p, c_int32, c_int64, c_int64, c_int64, c_void_p,
                               dq_format, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                               c_void_p]),
    "dq_w4a4_gemm_workspace_bytes": (c_size_t, [c_int64, c_int64, c_int64]),
    "dq_w4a4_gemm": (c_int32, [c_void_p, c_void_p, c_void_p, c_int64, c_void_p, c_void_p,
                               c_void_p, c_int64, c_int64, dq_format, c_void_p, c_int64,
                               c_void_p, c_size_t, c_void_p]),
    "dq_w4a4_linear_workspace_bytes": (c_size_t, [c_int64, c_int64, c_int64, dq_format]),
    "dq_w4a4_linear": (c_int32, [c_void_p, c_int32, c_int64, c_int64, c_int64, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_int64, dq_format, c_void_p,
                                 c_int64, c_void_p, c_size_t, c_void_p]),
    "dq_encode": (c_int32, [c_void_p, c_int64, c_int32, c_void_p, c_void_p]),
    "dq_decode": (c_int32, [c_void_p, c_int64, c_int32, c_void_p, c_void_p]),
    "dq_last_device_error": (c_int32, [c_void_p]),
    "dq_set_timing_events": (c_int32, [ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p),
                                       c_int32]),
    "dq_timing_events_used": (c_int32, []),
    "dq_kernel_launches": (c_int64, []),
}


_LIB = None


def get() -> ctypes.CDLL:
    """The process-wide handle of libdq.so (loaded on first use)."""
    global _LIB
    if _LIB is None:
        _LIB = load()
    return _LIB


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            "libdq.so is not built (expected at %s); run "
            "`python -m calibration_free_dual_b200.build`" % path)
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
