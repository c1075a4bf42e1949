"""Torch-tensor marshalling for the libdq C ABI (no computation happens here).

Each helper checks shapes/dtypes, allocates outputs and the workspace with torch on the
input's device, and passes raw pointers and the current CUDA stream to the C entry point of
the same role. The returned dicts keep the workspace alive until the caller drops them.
"""
from __future__ import annotations

import ctypes
from typing import Iterable

import torch

from . import _lib

FORMATS = {
    "INT4": (_lib.DQ_INT4, 128), "INT4_G128": (_lib.DQ_INT4, 128),
    "INT4_G64": (_lib.DQ_INT4, 64), "MXINT4": (_lib.DQ_MXINT4, 32),
    "MXFP4": (_lib.DQ_MXFP4, 32), "NVFP4": (_lib.DQ_NVFP4, 16),
    "INT8": (_lib.DQ_INT8, 128), "INT8_G128": (_lib.DQ_INT8, 128),
    "INT8_G64": (_lib.DQ_INT8, 64), "MXINT8": (_lib.DQ_MXINT8, 32),
}
_KIND_NAMES = {"INT4": _lib.DQ_INT4, "MXINT4": _lib.DQ_MXINT4, "MXFP4": _lib.DQ_MXFP4,
               "NVFP4": _lib.DQ_NVFP4, "INT8": _lib.DQ_INT8, "MXINT8": _lib.DQ_MXINT8}
_BF16_SCALES = (_lib.DQ_INT4, _lib.DQ_INT8)


def _code_cols(f, n: int) -> int:
    """Bytes of element codes per row: two 4-bit codes per byte, one 8-bit code."""
    return n if f.kind in (_lib.DQ_INT8, _lib.DQ_MXINT8) else n // 2


class DQError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        name = _lib.get().dq_status_string(self.status).decode()
        super().__init__("%s%s" % (name, (": " + what) if what else ""))


def _check(status: int, what: str = "") -> None:
    if status != _lib.DQ_OK:
        raise DQError(status, what)


def fmt_of(fmt) -> _lib.dq_format:
    """'NVFP4' | (kind, group) | object with .kind/.group (kind as name or number)."""
    if isinstance(fmt, _lib.dq_format):
        return fmt
    if isinstance(fmt, str):
        k, g = FORMATS[fmt]
    elif isinstance(fmt, tuple):
        k, g = fmt
    else:
        k, g = fmt.kind, fmt.group
    if isinstance(k, str):
        k = _KIND_NAMES[k]
    return _lib.dq_format(int(k), int(g))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return _lib.DQ_BF16
    if t.dtype == torch.float32:
        return _lib.DQ_F32
    raise TypeError("inputs must be bfloat16 or float32, got %s" % t.dtype)


def _p(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need_cuda(t: torch.Tensor, name: str) -> None:
    if not (isinstance(t, torch.Tensor) and t.is_cuda):
        raise TypeError("%s must be a CUDA tensor (there is no CPU path)" % name)


def solve_outputs(m: int, n: int, fmt, iters: int, device) -> dict:
    f = fmt_of(fmt)
    B = f.group
    sdt = torch.int16 if f.kind in _BF16_SCALES else torch.uint8
    return dict(
        q_packed=torch.empty((m, _code_cols(f, n)), dtype=torch.uint8, device=device),
        r=torch.empty((m, n // B), dtype=torch.float32, device=device),
        c=torch.empty((n,), dtype=torch.float32, device=device),
        block_scales=torch.empty((m, n // B), dtype=sdt, device=device),
        tensor_scale=torch.empty((1,), dtype=torch.float32, device=device),
        mse=torch.empty((iters + 1,), dtype=torch.float64, device=device),
    )


UPDATES = {"both": _lib.DQ_UPDATE_BOTH, "row": _lib.DQ_UPDATE_ROW_ONLY,
           "col": _lib.DQ_UPDATE_COL_ONLY}


def solve_batched(Ws: Iterable[torch.Tensor], fmt, iters: int, r0s=None, c0s=None,
                  stream=None, outs=None, workspace: torch.Tensor | None = None,
                  update: str = "both", qchange: bool = False) -> list:
    """dq_solve_batched over a list of 2-D CUDA matrices (all bf16 or all fp32).

    update: "both", "row" (r only) or "col" (c only); qchange: also return the Q-change
    trace ("qchange", [iters+1] fp64). Either option goes through dq_solve_batched_ex."""
    Ws = list(Ws)
    if not Ws:
        return []
    f = fmt_of(fmt)
    dt = _dtype_code(Ws[0])
    count = len(Ws)
    mats = (_lib.dq_matrix * count)()
    results = outs if outs is not None else []
    ms = (ctypes.c_int64 * count)()
    ns = (ctypes.c_int64 * count)()
    for i, W in enumerate(Ws):
        _need_cuda(W, "W")
        if W.dim() != 2 or W.stride(1) != 1 or _dtype_code(W) != dt:
            raise ValueError("each W must be 2-D, row-major, and share one dtype")
        m, n = W.shape
        ms[i], ns[i] = m, n
        if outs is None:
            results.append(solve_outputs(m, n, f, iters, W.device))
        o = results[i]
        r0 = r0s[i] if r0s is not None else None
        c0 = c0s[i] if c0s is not None else None
        mats[i] = _lib.dq_matrix(
            W.data_ptr(), m, n, W.stride(0),
            r0.data_ptr() if r0 is not None else None,
            c0.data_ptr() if c0 is not None else None,
            o["q_packed"].data_ptr(), o["r"].data_ptr(), o["c"].data_ptr(),
            o["block_scales"].data_ptr(), o["tensor_scale"].data_ptr(), o["mse"].data_ptr())
    lib = _lib.get()
    if update not in UPDATES:
        raise ValueError("update must be one of %s" % sorted(UPDATES))
    opts = None
    if update != "both" or qchange:
        qptrs = None
        if qchange:
            for o in results:
                o["qchange"] = torch.empty((iters + 1,), dtype=torch.float64,
                                           device=Ws[0].device)
            qptrs = (ctypes.c_void_p * count)(*[o["qchange"].data_ptr() for o in results])
        opts = _lib.dq_solve_options(UPDATES[update], qptrs)
    need = lib.dq_solve_workspace_bytes_ex(count, ms, ns, f, iters,
                                           ctypes.byref(opts) if opts is not None else None)
    if need == 0:
        raise DQError(_lib.DQ_ERR_UNSUPPORTED, "no workspace size for these shapes")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty((need,), dtype=torch.uint8, device=Ws[0].device)
    if opts is None:
        _check(lib.dq_solve_batched(mats, count, dt, f, iters, _p(workspace), need,
                                    _stream_ptr(stream)), "dq_solve_batched")
    else:
        _check(lib.dq_solve_batched_ex(mats, count, dt, f, iters, ctypes.byref(opts),
                                       _p(workspace), need, _stream_ptr(stream)),
               "dq_solve_batched_ex")
    for o in results:
        o["_workspace"] = workspace
    return results


def solve(W: torch.Tensor, fmt, iters: int, r0=None, c0=None, stream=None) -> dict:
    """Single-matrix solve through dq_solve."""
    _need_cuda(W, "W")
    if W.dim() != 2 or W.stride(1) != 1:
        raise ValueError("W must be 2-D row-major")
    f = fmt_of(fmt)
    m, n = W.shape
    o = solve_outputs(m, n, f, iters, W.device)
    lib = _lib.get()
    ms, ns = (ctypes.c_int64 * 1)(m), (ctypes.c_int64 * 1)(n)
    need = lib.dq_solve_workspace_bytes(1, ms, ns, f, iters)
    if need == 0:
        raise DQError(_lib.DQ_ERR_UNSUPPORTED if n % f.group == 0 else _lib.DQ_ERR_SHAPE,
                      "no workspace size for this shape")
    ws = torch.empty((need,), dtype=torch.uint8, device=W.device)
    _check(lib.dq_solve(_p(W), _dtype_code(W), m, n, W.stride(0), f, iters, _p(r0), _p(c0),
                        _p(o["q_packed"]), _p(o["r"]), _p(o["c"]), _p(o["block_scales"]),
                        _p(o["tensor_scale"]), _p(o["mse"]), _p(ws), need,
                        _stream_ptr(stream)), "dq_solve")
    o["_workspace"] = ws
    return o


def act_quant(X: torch.Tensor, fmt, c: torch.Tensor | None = None, stream=None) -> dict:
    """dq_act_quant: quantize fl32(X * c) per (token, block)."""
    _need_cuda(X, "X")
    if X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be 2-D row-major")
    f = fmt_of(fmt)
    T, n = X.shape
    B = f.group
    sdt = torch.int16 if f.kind in _BF16_SCALES else torch.uint8
    o = dict(x_packed=torch.empty((T, _code_cols(f, n)), dtype=torch.uint8, device=X.device),
             scales=torch.empty((T, n // B), dtype=sdt, device=X.device),
             tensor_scale=torch.empty((1,), dtype=torch.float32, device=X.device))
    lib = _lib.get()
    need = lib.dq_act_quant_workspace_bytes(T, n, f)
    ws = torch.empty((max(need, 16),), dtype=torch.uint8, device=X.device)
    if c is not None:
        _need_cuda(c, "c")
    _check(lib.dq_act_quant(_p(X), _dtype_code(X), T, n, X.stride(0), _p(c), f,
                            _p(o["x_packed"]), _p(o["scales"]), _p(o["tensor_scale"]), _p(ws),
                            ws.numel(), _stream_ptr(stream)), "dq_act_quant")
    o["_workspace"] = ws
    return o


def w4a4_gemm(x: dict, w: dict, fmt="NVFP4", stream=None,
              workspace: torch.Tensor | None = None) -> torch.Tensor:
    """dq_w4a4_gemm: y[T, N] from act_quant's output `x` (x_packed, scales, tensor_scale)
    and a solve's output `w` (q_packed, block_scales, tensor_scale)."""
    f = fmt_of(fmt)
    xq, xs, xst = x["x_packed"], x["scales"], x["tensor_scale"]
    wq, ws, wst = w["q_packed"], w["block_scales"], w["tensor_scale"]
    for t, name in ((xq, "x_packed"), (xs, "scales"), (wq, "q_packed"), (ws, "block_scales")):
        _need_cuda(t, name)
        if not t.is_contiguous():
            raise ValueError(name + " must be contiguous")
    T, N, K = xq.shape[0], wq.shape[0], xq.shape[1] * 2
    if wq.shape[1] * 2 != K:
        raise ValueError("activation and weight K differ")
    y = torch.empty((T, N), dtype=torch.float32, device=xq.device)
    lib = _lib.get()
    need = lib.dq_w4a4_gemm_workspace_bytes(T, N, K)
    if need == 0:
        raise DQError(_lib.DQ_ERR_SHAPE, "K must be a multiple of 64")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty((need,), dtype=torch.uint8, device=xq.device)
    _check(lib.dq_w4a4_gemm(_p(xq), _p(xs), _p(xst), T, _p(wq), _p(ws), _p(wst), N, K, f,
                            _p(y), N, _p(workspace), need, _stream_ptr(stream)),
           "dq_w4a4_gemm")
    return y


def w4a4_linear(X: torch.Tensor, w: dict, c: torch.Tensor | None = None, fmt="NVFP4",
                stream=None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """dq_w4a4_linear: y[T, N] = quantized fl32(X * c) times a solve's output `w`
    (q_packed, block_scales, tensor_scale), the activation quantized in the GEMM's layouts."""
    _need_cuda(X, "X")
    if X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be 2-D row-major")
    f = fmt_of(fmt)
    wq, ws, wst = w["q_packed"], w["block_scales"], w["tensor_scale"]
    for t, name in ((wq, "q_packed"), (ws, "block_scales")):
        _need_cuda(t, name)
        if not t.is_contiguous():
            raise ValueError(name + " must be contiguous")
    T, K = X.shape
    N = wq.shape[0]
    if wq.shape[1] * 2 != K:
        raise ValueError("activation and weight K differ")
    if c is not None:
        _need_cuda(c, "c")
    y = torch.empty((T, N), dtype=torch.float32, device=X.device)
    lib = _lib.get()
    need = lib.dq_w4a4_linear_workspace_bytes(T, N, K, f)
    if need == 0:
        raise DQError(_lib.DQ_ERR_SHAPE, "NVFP4 and K a multiple of 64 required")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty((need,), dtype=torch.uint8, device=X.device)
    _check(lib.dq_w4a4_linear(_p(X), _dtype_code(X), T, K, X.stride(0), _p(c), _p(wq), _p(ws),
                              _p(wst), N, f, _p(y), N, _p(workspace), need,
                              _stream_ptr(stream)), "dq_w4a4_linear")
    return y


_CODE_DTYPE = {_lib.DQ_CODEC_BF16: torch.int16}


def encode(x: torch.Tensor, codec: int, stream=None) -> torch.Tensor:
    _need_cuda(x, "x")
    x = x.contiguous().to(torch.float32)
    codes = torch.empty(x.shape, dtype=_CODE_DTYPE.get(codec, torch.uint8), device=x.device)
    _check(_lib.get().dq_encode(_p(x), x.numel(), codec, _p(codes), _stream_ptr(stream)),
           "dq_encode")
    return codes


def decode(codes: torch.Tensor, codec: int, stream=None) -> torch.Tensor:
    _need_cuda(codes, "codes")
    codes = codes.contiguous()
    x = torch.empty(codes.shape, dtype=torch.float32, device=codes.device)
    _check(_lib.get().dq_decode(_p(codes), codes.numel(), codec, _p(x), _stream_ptr(stream)),
           "dq_decode")
    return x


def last_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return int(_lib.get().dq_last_device_error(_stream_ptr(stream)))
