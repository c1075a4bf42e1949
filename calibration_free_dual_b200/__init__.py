"""DualQuant dual-scale solver for NVIDIA B200 (sm_100a).

The C library `libdq.so` (include/dq.h) does all the work in hand-written CUDA kernels;
this package only loads it and marshals torch tensors into its calls. There is no CPU
fallback: the first use raises ImportError if the library is missing, and every call needs
CUDA tensors.

The C ABI is reachable under its own names (`dq_solve`, `dq_solve_batched`,
`dq_act_quant`, ... taking raw pointers); the helpers in `api` allocate outputs and the
workspace with torch and call them.
"""
from . import _lib
from ._lib import (DQ_OK, DQ_INT4, DQ_MXINT4, DQ_MXFP4, DQ_NVFP4, DQ_INT8,  # noqa: F401
                   DQ_MXINT8, DQ_F32, DQ_BF16, DQ_CODEC_INT4, DQ_CODEC_E2M1, DQ_CODEC_E4M3,
                   DQ_CODEC_E8M0, DQ_CODEC_BF16, DQ_CODEC_INT8,
                   DQ_UPDATE_BOTH, DQ_UPDATE_ROW_ONLY, DQ_UPDATE_COL_ONLY,
                   dq_format, dq_matrix, dq_solve_options)
from .api import (DQError, FORMATS, fmt_of, solve, solve_batched, act_quant, encode,  # noqa: F401
                  decode, last_device_error, w4a4_gemm,
                  w4a4_linear)


def __getattr__(name):
    # the C entry points, loaded from libdq.so on first access
    if name in _lib.SIGNATURES:
        return getattr(_lib.get(), name)
    if name == "lib":
        return _lib.get()
    raise AttributeError(name)
