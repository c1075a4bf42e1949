"""Parity of the CUDA activation rescale + block quantization with the oracle (B200).

Every decision in this path is taken on the same binary32 values on both sides (the
product X*c, the block maximum, fl32(a/q_max), the scale projection and fl32(x*1/d)), so
codes and scale codes must agree bit for bit, and the SQNRs computed from them agree.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import formats as F
from oracle import solver as S
from oracle.actquant import act_quant as ora_act, dequant, sqnr
from tests._parity import oracle_format

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dq():
    import calibration_free_dual_b200 as pkg
    return pkg


def _gpu_act(dq, X, fmt_name, c):
    o = dq.act_quant(X.cuda(), fmt_name, None if c is None else torch.from_numpy(c).cuda())
    torch.cuda.synchronize()
    assert dq.last_device_error() == 0
    return {k: v.cpu().numpy() for k, v in o.items() if not k.startswith("_")}


def _check(h, ora, fmt):
    codes = F.unpack_codes(h["x_packed"], fmt.bits)
    np.testing.assert_array_equal(codes, ora["codes"])
    sc = h["scales"].view(np.uint16) if fmt.scale == "bf16" else h["scales"]
    np.testing.assert_array_equal(sc.astype(np.int64), ora["scale_codes"].astype(np.int64))
    if fmt.kind == "NVFP4":
        assert np.float32(h["tensor_scale"][0]) == ora["s_t"]


def _decode_gpu(h, fmt):
    codes = F.unpack_codes(h["x_packed"], fmt.bits)
    q = F.decode_elem(codes, fmt)
    sc = h["scales"].view(np.uint16) if fmt.scale == "bf16" else h["scales"]
    s_t = h["tensor_scale"][0] if fmt.kind == "NVFP4" else None
    d = F.decode_scale(sc, fmt, s_t).astype(np.float64)
    if fmt.scale == "bf16":
        d = np.where(sc == 0, 0.0, d)
    return dequant(d, q, fmt.block)


@pytest.mark.parametrize("fmt_name", ["NVFP4", "INT4", "INT4_G64", "MXFP4", "MXINT4", "INT8",
                                      "INT8_G64", "MXINT8"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_act_quant_bit_exact(dq, fmt_name, dtype):
    rng = np.random.default_rng(3)
    T, n = 77, 1280                       # ragged last 512-channel strip, odd token count
    X = rng.standard_normal((T, n)).astype(np.float32)
    X[:, rng.choice(n, 4, replace=False)] *= 50
    X[5, :] = 0.0                          # an all-zero token row
    c = rng.uniform(0.25, 3.0, n).astype(np.float32)
    Xt = torch.from_numpy(X)
    if dtype == "bf16":
        Xt = Xt.to(torch.bfloat16)
    fmt = oracle_format(fmt_name)
    Xn = Xt.float().numpy()
    for cc in (c, None):
        h = _gpu_act(dq, Xt, fmt_name, cc)
        ora = ora_act(Xn, fmt, cc)
        _check(h, ora, fmt)


def test_act_quant_config_sqnr(dq):
    """8192 tokens x 4096 channels with six x50 channels; c from the oracle's MXFP4 solve of
    a 1024x4096 k_proj drawn with the Student-t recipe. SQNR with and without c agree."""
    cfg = wl.ACT_KPROJ
    Wk = wl.weight_host(cfg, 0, 1)
    c = S.solve(Wk.float().numpy().astype(np.float64), oracle_format("MXFP4"), cfg.iters)["c"]
    X = wl.act_host()
    Xn = X.float().numpy()
    for fmt_name in ("NVFP4", "INT4"):
        fmt = oracle_format(fmt_name)
        res = {}
        for tag, cc in (("with_c", c), ("without_c", None)):
            h = _gpu_act(dq, X, fmt_name, cc)
            ora = ora_act(Xn, fmt, cc)
            _check(h, ora, fmt)
            s_gpu = sqnr(ora["xt"], _decode_gpu(h, fmt))
            s_ora = sqnr(ora["xt"], dequant(ora["d"], ora["q"], fmt.block))
            assert abs(s_gpu - s_ora) <= 1e-4
            res[tag] = s_gpu
        assert all(np.isfinite(v) and v > 5 for v in res.values()), res


@pytest.mark.parametrize("fmt_name", ["MXFP4", "NVFP4", "INT4"])
@pytest.mark.parametrize("bad", [float("inf"), float("-inf"), float("nan")])
def test_act_nonfinite_reported(dq, fmt_name, bad):
    """A non-finite channel anywhere in a block (first, middle, last element) is reported,
    also through the NVFP4 amax pass and through the linear path."""
    for col in (0, 37, 127):
        X = torch.randn(8, 128)
        X[2, col] = bad
        dq.act_quant(X.cuda(), fmt_name)
        assert dq.last_device_error() == 5
    assert dq.last_device_error() == 0


@pytest.mark.parametrize("fmt_name", ["NVFP4", "INT4", "MXFP4", "INT8", "MXINT8"])
def test_act_quant_offset_codes_and_strided_x(dq, fmt_name):
    """Codes written to a buffer that is only as aligned as the interface requires (4 bytes
    for the 4-bit formats, 8 for the 8-bit ones: one store per lane is split in two) and X
    read through a row pitch larger than its width give the same codes as the oracle."""
    import ctypes
    from calibration_free_dual_b200 import _lib
    from calibration_free_dual_b200.api import fmt_of
    rng = np.random.default_rng(11)
    T, n, ld = 40, 1536, 1600
    Xfull = torch.from_numpy(rng.standard_normal((T, ld)).astype(np.float32)).to(torch.bfloat16)
    Xd = Xfull.cuda()
    X = Xd[:, :n]
    c = rng.uniform(0.5, 2.0, n).astype(np.float32)
    fmt = oracle_format(fmt_name)
    f = fmt_of(fmt_name)
    cols = n if fmt.bits == 8 else n // 2
    off = 8 if fmt.bits == 8 else 4
    buf = torch.zeros(T * cols + 64, dtype=torch.uint8, device="cuda")
    base = buf.data_ptr() + off
    sdt = torch.int16 if fmt.scale == "bf16" else torch.uint8
    scales = torch.empty((T, n // fmt.block), dtype=sdt, device="cuda")
    ts = torch.empty((1,), dtype=torch.float32, device="cuda")
    lib = _lib.get()
    ws = torch.empty((lib.dq_act_quant_workspace_bytes(T, n, f),), dtype=torch.uint8,
                     device="cuda")
    cd = torch.from_numpy(c).cuda()
    st = lib.dq_act_quant(ctypes.c_void_p(X.data_ptr()), _lib.DQ_BF16, T, n, ld,
                          ctypes.c_void_p(cd.data_ptr()), f, ctypes.c_void_p(base),
                          ctypes.c_void_p(scales.data_ptr()), ctypes.c_void_p(ts.data_ptr()),
                          ctypes.c_void_p(ws.data_ptr()), ws.numel(), None)
    assert st == 0
    torch.cuda.synchronize()
    assert dq.last_device_error() == 0
    raw = buf.cpu().numpy()
    assert not raw[:off].any() and not raw[off + T * cols:].any()   # nothing outside
    h = dict(x_packed=raw[off:off + T * cols].reshape(T, cols), scales=scales.cpu().numpy(),
             tensor_scale=ts.cpu().numpy())
    ora = ora_act(Xfull.float().numpy()[:, :n], fmt, c)
    _check(h, ora, fmt)
