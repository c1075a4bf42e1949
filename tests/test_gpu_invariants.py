"""Exact symmetries of the BCD solve, checked on the CUDA path itself (B200).

Each holds bit for bit in the kernels' binary32 arithmetic, independently of the oracle:
  * W -> 2^k W: every product and sum of the solve scales by a power of two, so the codes and
    c are unchanged, the decoded block scales scale by 2^k and the normalised trace is equal
    (the DualQuant model diag(r) Q diag(c) is homogeneous in r);
  * W -> -W: the element grids are symmetric and rounding is to nearest even, so the codes
    negate and every scale and the trace are unchanged;
  * column strips: r and c couple only the columns of one format block (r-step) or the rows
    of one column (c-step), so a strip of whole tiles solved on its own gives the same
    state as inside the full matrix (formats without a per-tensor scale).
"""
import numpy as np
import pytest
import torch

from oracle import formats as F
from tests._parity import oracle_format, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dq():
    import calibration_free_dual_b200 as pkg
    return pkg


def _w(seed, m, n):
    rng = np.random.default_rng(seed)
    w = rng.standard_t(4, (m, n)) * 0.014
    w[:, rng.choice(n, 3, replace=False)] *= 10.0
    return torch.from_numpy(w.astype(np.float32)).to(torch.bfloat16)


def _solve(dq, W, fmt_name, iters):
    out = dq.solve(W, fmt_name, iters)
    torch.cuda.synchronize()
    assert dq.last_device_error() == 0
    return to_host(out)


def _values(h, fmt):
    return F.decode_elem(F.unpack_codes(h["q_packed"], fmt.bits), fmt)


FMTS = ["NVFP4", "MXFP4", "MXINT4", "INT4", "INT4_G64", "MXINT8", "INT8"]


@pytest.mark.parametrize("fmt_name", FMTS)
@pytest.mark.parametrize("k", [4, -6])
def test_power_of_two_scaling(dq, fmt_name, k):
    W = _w(5, 256, 512)
    a = _solve(dq, W.cuda(), fmt_name, 6)
    b = _solve(dq, (W.float() * 2.0 ** k).to(torch.bfloat16).cuda(), fmt_name, 6)
    np.testing.assert_array_equal(a["q_packed"], b["q_packed"])
    np.testing.assert_array_equal(a["r"].astype(np.float64) * 2.0 ** k, b["r"].astype(np.float64))
    np.testing.assert_array_equal(a["c"], b["c"])
    np.testing.assert_array_equal(a["mse"], b["mse"])
    if fmt_name == "NVFP4":
        np.testing.assert_array_equal(a["block_scales"], b["block_scales"])
        assert b["tensor_scale"][0] == np.float32(a["tensor_scale"][0] * 2.0 ** k)


@pytest.mark.parametrize("fmt_name", FMTS)
def test_sign_flip(dq, fmt_name):
    W = _w(6, 192, 384)
    fmt = oracle_format(fmt_name)
    a = _solve(dq, W.cuda(), fmt_name, 6)
    b = _solve(dq, (-W).cuda(), fmt_name, 6)
    np.testing.assert_array_equal(_values(a, fmt), -_values(b, fmt))
    for key in ("r", "block_scales", "c", "mse"):
        np.testing.assert_array_equal(a[key], b[key], err_msg=key)


@pytest.mark.parametrize("fmt_name", ["MXFP4", "MXINT4", "INT4", "INT4_G64", "MXINT8"])
def test_column_strip_solves_alone(dq, fmt_name):
    """Columns [256, 512) of a 300 x 1024 matrix (whole 128-column tiles at both widths) solved
    as a strided view of their own: identical codes, block scales and c."""
    fmt = oracle_format(fmt_name)
    W = _w(7, 300, 1024).cuda()
    full = _solve(dq, W, fmt_name, 8)
    part = _solve(dq, W[:, 256:512], fmt_name, 8)
    per_byte = 8 // fmt.bits
    np.testing.assert_array_equal(full["q_packed"][:, 256 // per_byte:512 // per_byte],
                                  part["q_packed"])
    B = fmt.block
    for key in ("r", "block_scales"):
        np.testing.assert_array_equal(full[key][:, 256 // B:512 // B], part[key], err_msg=key)
    np.testing.assert_array_equal(full["c"][256:512], part["c"])
