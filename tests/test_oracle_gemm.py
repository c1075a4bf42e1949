"""Pins for the oracle's W4A4 GEMM (CPU only).

* brute force: explicit loops over codes, scales and the E2M1 / E4M3 tables on tiny inputs;
* the dual-scale model: when the rescaled activation is exactly on its grid, the GEMM of
  the two quantized operands equals W_hat x with W_hat = diag(r) Q diag(c) (the column
  scale has moved into the activation, the ai4snews summary paragraph 3 direction);
* scaling: the output scales with the product of the two tensor scales.
"""
import numpy as np

from oracle import formats as F
from oracle import gemm as G
from oracle import solver as S
from oracle.actquant import act_quant

NV = F.make_format("NVFP4")


def _rand_operand(rng, rows, n, zero_block=False):
    codes = rng.integers(0, 16, (rows, n)).astype(np.uint8)
    sc = rng.integers(1, 127, (rows, n // 16)).astype(np.uint8)
    if zero_block:
        sc[0, 0] = 0
        codes[0, :16] = 0
    return codes, sc


def test_gemm_brute_force():
    rng = np.random.default_rng(0)
    xc, xs = _rand_operand(rng, 3, 32, zero_block=True)
    wc, ws = _rand_operand(rng, 2, 32)
    sx, sw = np.float32(0.375), np.float32(1.25)
    got = G.w4a4_gemm(xc, xs, sx, wc, ws, sw, NV)
    e2m1 = lambda c: (-1.0 if c & 8 else 1.0) * F.E2M1_MAG[c & 7]
    for t in range(3):
        for i in range(2):
            acc = 0.0
            for j in range(32):
                dx = 0.0 if xs[t, j // 16] == 0 else float(sx) * F.E4M3_POS[xs[t, j // 16]]
                dw = float(sw) * F.E4M3_POS[ws[i, j // 16]]
                acc += dx * e2m1(int(xc[t, j])) * dw * e2m1(int(wc[i, j]))
            assert abs(got[t, i] - acc) <= 1e-12 * max(1.0, abs(acc)), (t, i, got[t, i], acc)


def test_gemm_is_w_hat_x_when_the_activation_is_on_its_grid():
    """Take a dual-scale weight W_hat = diag(r) Q diag(c) (E4M3 block scales r, power-of-two
    column scales c) and an activation x whose rescale c * x lies exactly on the activation
    grid; the GEMM of the two quantized operands, which never sees c, is then W_hat x."""
    rng = np.random.default_rng(1)
    m, n, T = 8, 64, 5
    s_w = np.float32(0.01)
    wq_codes = rng.integers(0, 16, (m, n)).astype(np.uint8)
    wr_codes = rng.integers(1, 127, (m, n // 16)).astype(np.uint8)
    c = (2.0 ** rng.integers(-2, 3, n)).astype(np.float32)
    r = F.decode_scale(wr_codes, NV, s_w).astype(np.float64)
    w_hat = S.reconstruct(F.decode_elem(wq_codes, NV), r, c, NV.block)
    # activation on the grid after rescaling: 6 * 2^k * E2M1 values per block, so the block
    # maximum is 6 * 2^k and the quantizer reproduces every value exactly
    xt = np.zeros((T, n))
    for t in range(T):
        for b in range(n // 16):
            q = F.E2M1_MAG[rng.integers(0, 8, 16)] * rng.choice([-1.0, 1.0], 16)
            q[0] = 6.0
            xt[t, b * 16:(b + 1) * 16] = q * 2.0 ** int(rng.integers(-3, 3))
    X = (xt / c[None, :]).astype(np.float32)
    assert np.all((X * c[None, :]).astype(np.float64) == xt)
    a = act_quant(X, NV, c)
    np.testing.assert_array_equal(G.dequantize(a["codes"], a["scale_codes"], NV, a["s_t"],
                                               zero_code_is_zero=True), xt)
    y = G.w4a4_gemm(a["codes"], a["scale_codes"], a["s_t"], wq_codes, wr_codes, s_w, NV)
    ref = X.astype(np.float64) @ w_hat.T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)


def test_gemm_scales_with_the_tensor_scales():
    rng = np.random.default_rng(2)
    xc, xs = _rand_operand(rng, 4, 64)
    wc, ws = _rand_operand(rng, 3, 64)
    y1 = G.w4a4_gemm(xc, xs, np.float32(1.0), wc, ws, np.float32(1.0), NV)
    y2 = G.w4a4_gemm(xc, xs, np.float32(0.5), wc, ws, np.float32(4.0), NV)
    np.testing.assert_array_equal(y2, 2.0 * y1)
