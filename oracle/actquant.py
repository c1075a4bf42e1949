"""Activation rescale by the solver's column scales + 4-bit block quantization (oracle).

DualQuant's column scales double as per-channel activation rescalings applied before the
activation quantizer, with no calibration data ("DualQuant: Dual-scale Calibration-free
Weight-and-Activation Quantization for LLMs", Abstract; appendix Table 11 "Activation
quantization (incl. beta)"; appendix Table 6 measures the activation SQNR with and without
the rescaling; the ai4snews summary, paragraph 3).

Direction: with W_hat = diag(r) Q diag(c), W_hat x = diag(r) Q (c * x), so the activation
the quantized GEMM consumes is c * x (elementwise); that product is what is quantized.
Blocks are B consecutive channels of one token row.
"""
from __future__ import annotations

import numpy as np

from .formats import Format, round_elem, project_scale, nvfp4_tensor_scale


def rescale(X: np.ndarray, c=None) -> np.ndarray:
    """x~ = fl32(X * c) per channel (binary32 product), or X itself without c."""
    X32 = np.asarray(X, dtype=np.float32)
    if c is None:
        return X32.copy()
    return (X32 * np.asarray(c, dtype=np.float32)[None, :]).astype(np.float32)


def act_quant(X, fmt: Format, c=None):
    """Quantize fl32(X * c) to 4-bit codes with per-(token, block) scales.

    Returns dict: codes [T, n] uint8, scale_codes [T, n/B], d (decoded block scales,
    binary32, 0 for an all-zero block), s_t (NVFP4), xt (the rescaled binary32 input),
    q (element values, float64)."""
    xt = rescale(X, c)
    T, n = xt.shape
    B = fmt.block
    if n % B:
        raise ValueError("channels must be a multiple of the block length")
    a = np.max(np.abs(xt.reshape(T, n // B, B)), axis=2)                   # binary32, exact
    s_t = None
    if fmt.kind == "NVFP4":
        s_t = nvfp4_tensor_scale(float(np.max(a)) if a.size else 0.0)
    nz = a > 0
    v = (a / np.float32(fmt.qmax)).astype(np.float32)
    v = np.where(nz, v, np.float32(1.0)).astype(np.float32)
    sc, d = project_scale(v, fmt, s_t)
    sc = np.where(nz, sc, 0).astype(sc.dtype)
    d = np.where(nz, d, np.float32(0.0)).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(nz, np.float32(1.0) / np.where(nz, d, np.float32(1.0)),
                       np.float32(0.0)).astype(np.float32)
    x = (xt * np.repeat(inv, B, axis=1)).astype(np.float32)
    codes, q = round_elem(x, fmt)
    zero = ~np.repeat(nz, B, axis=1)
    codes = np.where(zero, 0, codes).astype(np.uint8)
    q = np.where(zero, 0.0, q)
    return dict(codes=codes, scale_codes=sc, d=d, s_t=s_t, xt=xt, q=q)


def dequant(d: np.ndarray, q: np.ndarray, B: int) -> np.ndarray:
    return np.repeat(np.asarray(d, dtype=np.float64), B, axis=1) * q


def sqnr(xt: np.ndarray, xhat: np.ndarray) -> float:
    """10 log10( sum x~^2 / sum (x~ - x_hat)^2 ), binary64."""
    xt = np.asarray(xt, dtype=np.float64)
    err = float(np.sum((xt - xhat) ** 2))
    sig = float(np.sum(xt * xt))
    if err == 0.0:
        return float("inf")
    return 10.0 * np.log10(sig / err)
