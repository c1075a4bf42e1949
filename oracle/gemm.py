"""The W4A4 GEMM that consumes the solver's and the activation quantizer's outputs (oracle;
test only).

The DualQuant pages deploy the quantized model through a real packed W4A4 path (the
ai4snews summary, paragraph 4; the paper's appendix tables on the RTX 4090 path). With
W_hat = diag(r) Q diag(c) and the activation x~ = c * x quantized per (token, block) as
d * q_x, the layer output is

    y[t, i] = sum_j (d[t, b(j)] q_x[t, j]) (r[i, b(j)] q[i, j])

(c has moved into the activation, so the GEMM sees two block-scaled 4-bit operands). This
module is that sum, written as the plain definition: decode both operands to binary64 and
multiply.
"""
from __future__ import annotations

import numpy as np

from .formats import Format, decode_elem, decode_scale


def dequantize(codes: np.ndarray, scale_codes: np.ndarray, fmt: Format, s_t=None,
               zero_code_is_zero: bool = False) -> np.ndarray:
    """Element codes [rows, n] and block scale codes [rows, n/B] -> binary64 values.

    zero_code_is_zero: an activation block whose scale code is 0 stands for an all-zero
    block (the activation quantizer's convention); its values are 0."""
    q = decode_elem(codes, fmt)
    d = decode_scale(scale_codes, fmt, s_t).astype(np.float64)
    if zero_code_is_zero:
        d = np.where(np.asarray(scale_codes) == 0, 0.0, d)
    return q * np.repeat(d, fmt.block, axis=1)


def w4a4_gemm(x_codes, x_scale_codes, x_s_t, w_codes, w_scale_codes, w_s_t,
              fmt: Format) -> np.ndarray:
    """y [T, N] = dequant(X) @ dequant(W)^T in binary64."""
    X = dequantize(x_codes, x_scale_codes, fmt, x_s_t, zero_code_is_zero=True)
    W = dequantize(w_codes, w_scale_codes, fmt, w_s_t)
    return X @ W.T


def abs_products(x_codes, x_scale_codes, x_s_t, w_codes, w_scale_codes, w_s_t,
                 fmt: Format) -> np.ndarray:
    """sum_j |x_hat[t, j] w_hat[i, j]|: the scale of the rounding error of any summation
    order of y[t, i]."""
    X = dequantize(x_codes, x_scale_codes, fmt, x_s_t, zero_code_is_zero=True)
    W = dequantize(w_codes, w_scale_codes, fmt, w_s_t)
    return np.abs(X) @ np.abs(W).T
