"""Invariant and special-case pins for the oracle solve (CPU only).

* Theorem 1 (i) of the DualQuant paper (Figure 2 (b), Figure 3 (b)): the normalised MSE is
  monotone non-increasing over BCD iterations.
* c = 1 at iteration 0 is single-scale round-to-nearest (Figure 1 (b)), rebuilt here from
  torch's own bfloat16 / float8_e8m0fnu / float8_e4m3fn conversions.
* Fixed points, power-of-two scale and sign equivariance, row permutation, column-strip
  independence, resume from a saved state, and the direction of the activation rescale.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import formats as F
from oracle import solver as S
from oracle.actquant import act_quant, rescale

KINDS = ["INT4", "MXINT4", "MXFP4", "NVFP4", "INT8", "MXINT8"]


def _small(kind, seed=0, m=96, n=256):
    rng = np.random.default_rng(seed)
    W = rng.standard_t(4, (m, n)) * 0.014
    W[:, rng.choice(n, 3, replace=False)] *= 8.0
    return W.astype(np.float32).astype(np.float64)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("seed", range(3))
def test_theorem1_monotone_mse(kind, seed):
    fmt = F.make_format(kind)
    out = S.solve(_small(kind, seed), fmt, 20)
    m = out["mse"]
    assert np.all(m[1:] <= m[:-1] * (1 + 1e-12)), m
    assert m[-1] < m[0]                      # dual-scale beats single-scale here


def test_config1_dual_beats_single_and_traces():
    W = wl.weight_host(wl.CONFIGS[1], 0, 0).numpy().astype(np.float64)
    out = S.solve(W, F.make_format("INT4", 128), 20)
    m = out["mse"]
    assert np.all(np.diff(m) <= 1e-12 * m[:-1])
    assert m[0] / m[-1] > 4.0
    qc = out["qchange"]
    assert qc[-1] < qc[2]                    # Q-hat changes decay (Figure 2 (a))


def _rtn_reference(W, kind):
    """Single-scale RTN from torch conversions: block scale = format's scale of absmax/qmax."""
    fmt = F.make_format(kind)
    Wt = torch.from_numpy(W).to(torch.float32)
    m, n = W.shape
    a = Wt.reshape(m, n // fmt.block, fmt.block).abs().amax(dim=2)
    v = a / fmt.qmax
    if kind in ("INT4", "INT8"):
        s = v.to(torch.bfloat16).to(torch.float64)
    elif kind in ("MXINT4", "MXFP4", "MXINT8"):
        s = v.to(torch.float8_e8m0fnu).to(torch.float64)
    else:
        st = torch.tensor(float(a.max()), dtype=torch.float32) / 2688.0
        e = (v / st).to(torch.float8_e4m3fn).to(torch.float32)
        s = (st * e).to(torch.float64)
    x = Wt.to(torch.float64) / s.repeat_interleave(fmt.block, dim=1)
    if fmt.elem in ("int4", "int8"):
        q = torch.clamp(torch.round(x), -fmt.qmax, fmt.qmax)
    else:
        grid = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=torch.float64)
        d = (x.abs().unsqueeze(-1) - grid).abs()
        q = grid[d.argmin(-1)] * torch.sign(x)
    return s.numpy(), q.numpy(), x.numpy()


@pytest.mark.parametrize("kind", KINDS)
def test_iteration0_is_single_scale_rtn(kind):
    W = _small(kind, 11)
    fmt = F.make_format(kind)
    out = S.solve(W, fmt, 0)
    s_ref, q_ref, x_ref = _rtn_reference(W, kind)
    np.testing.assert_array_equal(out["r"].astype(np.float64), s_ref)
    np.testing.assert_array_equal(out["c"], np.ones(W.shape[1], np.float32))
    diff = out["q"] != q_ref
    if fmt.elem in ("int4", "int8"):
        mids = np.abs(np.abs(x_ref) - (np.floor(np.abs(x_ref)) + 0.5))
    else:
        g = F.E2M1_MAG
        mids = np.min(np.abs(np.abs(x_ref)[..., None] - (g[:-1] + g[1:]) / 2), axis=-1)
    # mismatches only where the quotient is on a rounding midpoint (ties / binary32 rounding)
    assert np.all(mids[diff] <= 1e-6 * np.maximum(np.abs(x_ref[diff]), 1))
    assert diff.mean() < 1e-3


@pytest.mark.parametrize("kind", KINDS)
def test_exact_model_is_a_fixed_point(kind):
    fmt = F.make_format(kind)
    rng = np.random.default_rng(3)
    m, n = 16, 4 * fmt.block
    s_t = np.float32(1.0 / 64)
    if fmt.scale == "bf16":
        r = (rng.integers(64, 128, (m, n // fmt.block)) / 2.0 ** 12).astype(np.float32)
    elif fmt.scale == "e8m0":
        r = (2.0 ** rng.integers(-9, -4, (m, n // fmt.block))).astype(np.float32)
    else:
        r = (s_t * F.E4M3_POS[rng.integers(40, 90, (m, n // fmt.block))]).astype(np.float32)
    qm = int(fmt.qmax)
    grid = np.arange(-qm, qm + 1) if fmt.elem != "e2m1" else np.concatenate(
        [-F.E2M1_MAG[:0:-1], F.E2M1_MAG])
    q = rng.choice(grid[grid != 0], (m, n)).astype(np.float64)
    c = (rng.integers(4, 16, n) / 8.0).astype(np.float32)     # few mantissa bits
    W = np.repeat(r.astype(np.float64), fmt.block, 1) * q * c.astype(np.float64)[None, :]
    assert np.all(W.astype(np.float32).astype(np.float64) == W)
    amax = float(s_t) * 2688.0 if kind == "NVFP4" else None
    out = S.solve(W, fmt, 5, r0=r, c0=c, amax=amax)
    assert np.all(out["mse"] == 0.0)
    np.testing.assert_array_equal(out["q"], q)
    np.testing.assert_array_equal(out["r"], r)
    np.testing.assert_array_equal(out["c"], c)


@pytest.mark.parametrize("kind", KINDS)
def test_power_of_two_equivariance(kind):
    W = _small(kind, 5, m=64, n=128)
    fmt = F.make_format(kind)
    a = S.solve(W, fmt, 6)
    b = S.solve(W * 2.0 ** 5, fmt, 6)
    np.testing.assert_array_equal(a["codes"], b["codes"])
    np.testing.assert_array_equal(a["r"] * np.float32(32.0), b["r"])
    np.testing.assert_array_equal(a["c"], b["c"])
    np.testing.assert_allclose(a["mse"], b["mse"], rtol=1e-12)


@pytest.mark.parametrize("kind", KINDS)
def test_sign_equivariance(kind):
    W = _small(kind, 6, m=64, n=128)
    fmt = F.make_format(kind)
    a = S.solve(W, fmt, 6)
    b = S.solve(-W, fmt, 6)
    np.testing.assert_array_equal(-a["q"], b["q"])
    np.testing.assert_array_equal(a["r"], b["r"])
    np.testing.assert_array_equal(a["c"], b["c"])


@pytest.mark.parametrize("kind", KINDS)
def test_row_permutation(kind):
    W = _small(kind, 7, m=64, n=128)
    fmt = F.make_format(kind)
    perm = np.random.default_rng(8).permutation(W.shape[0])
    a = S.solve(W, fmt, 6)
    b = S.solve(W[perm], fmt, 6)
    np.testing.assert_array_equal(a["codes"][perm], b["codes"])
    np.testing.assert_array_equal(a["r"][perm], b["r"])
    np.testing.assert_allclose(a["c"], b["c"], rtol=0, atol=0)


@pytest.mark.parametrize("kind", KINDS)
def test_column_strips_are_independent(kind):
    W = _small(kind, 9, m=48, n=256)
    fmt = F.make_format(kind)
    full = S.solve(W, fmt, 8)
    amax = float(np.max(np.abs(W)))
    B = fmt.block
    for b in range(W.shape[1] // B):
        cols = slice(b * B, (b + 1) * B)
        part = S.solve(W[:, cols], fmt, 8, amax=amax if kind == "NVFP4" else None)
        np.testing.assert_array_equal(part["codes"], full["codes"][:, cols])
        np.testing.assert_array_equal(part["r"][:, 0], full["r"][:, b])
        np.testing.assert_array_equal(part["c"], full["c"][cols])


@pytest.mark.parametrize("kind", KINDS)
def test_resume_from_saved_state(kind):
    W = _small(kind, 10, m=64, n=128)
    fmt = F.make_format(kind)
    full = S.solve(W, fmt, 8)
    head = S.solve(W, fmt, 5)
    amax = float(np.max(np.abs(W))) if kind == "NVFP4" else None
    tail = S.solve(W, fmt, 3, r0=head["r"], c0=head["c"], amax=amax)
    np.testing.assert_array_equal(tail["codes"], full["codes"])
    np.testing.assert_array_equal(tail["r"], full["r"])
    np.testing.assert_array_equal(tail["c"], full["c"])
    np.testing.assert_allclose(tail["mse"][1:], full["mse"][6:], rtol=1e-12)


def test_activation_rescale_direction_reproduces_w_hat_x():
    """W_hat x = diag(r) Q (c * x): the quantizer must see c * x, not x / c."""
    fmt = F.make_format("MXFP4")
    W = _small("MXFP4", 12, m=32, n=128)
    out = S.solve(W, fmt, 6)
    x = np.random.default_rng(13).standard_normal((5, 128)).astype(np.float32)
    what = S.reconstruct(out["q"], out["r"], out["c"], fmt.block)
    xt = rescale(x, out["c"]).astype(np.float64)
    rq = np.repeat(out["r"].astype(np.float64), fmt.block, 1) * out["q"]
    lhs = rq @ xt.T
    rhs = what @ x.astype(np.float64).T
    # the only error is the binary32 rounding of c * x (half an ulp per element)
    bound = (np.abs(rq) @ np.abs(xt).T) * 2.0 ** -23
    assert np.all(np.abs(lhs - rhs) <= bound)
    wrong = rq @ (x.astype(np.float64) / out["c"].astype(np.float64)).T
    assert np.max(np.abs(wrong - rhs)) > 1e3 * np.max(bound)


@pytest.mark.parametrize("kind", KINDS)
def test_act_quant_blocks_and_zero_blocks(kind):
    fmt = F.make_format(kind)
    rng = np.random.default_rng(14)
    X = rng.standard_normal((6, 2 * fmt.block)).astype(np.float32)
    X[2, :fmt.block] = 0.0
    c = rng.uniform(0.5, 2, 2 * fmt.block).astype(np.float32)
    out = act_quant(X, fmt, c)
    assert out["d"][2, 0] == 0 and np.all(out["codes"][2, :fmt.block] == 0)
    xt = out["xt"].astype(np.float64)
    # every non-zero block: absmax maps near the top of the grid, nothing beyond q_max
    a = np.abs(xt).reshape(6, 2, fmt.block).max(-1)
    assert np.all(np.abs(out["q"]) <= fmt.qmax)
    nz = a > 0
    ratio = a[nz] / out["d"][nz]
    assert np.all(ratio <= fmt.qmax * 1.5 + 1e-6) and np.all(ratio >= fmt.qmax / 2.1)


def test_sqnr_and_dequant_closed_forms():
    """SQNR = 10 log10(sum x^2 / sum (x - x_hat)^2): a reconstruction scaled by (1 - e) has
    SQNR -20 log10(e); exact reconstruction is infinite, a zero one is 0 dB. dequant puts the
    block scale d on each of the block's B elements."""
    from oracle.actquant import dequant, sqnr
    x = np.random.default_rng(21).standard_normal((4, 32))
    for e in (0.5, 0.1, 1e-3):
        assert sqnr(x, x * (1 - e)) == pytest.approx(-20 * np.log10(e), rel=1e-12)
    assert sqnr(x, x) == float("inf")
    assert sqnr(x, np.zeros_like(x)) == pytest.approx(0.0, abs=1e-12)
    d = np.array([[2.0, 0.5]])
    q = np.arange(8, dtype=np.float64).reshape(1, 8)
    np.testing.assert_array_equal(dequant(d, q, 4), [[0, 2, 4, 6, 2, 2.5, 3, 3.5]])
