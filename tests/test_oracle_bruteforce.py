"""Brute-force pins for the oracle's BCD steps on tiny matrices (CPU only).

Every closed-form / projected update must be the exact minimiser of its block of the
objective ||W - diag(r) Q diag(c)||^2 (the property Theorem 1 (i) of the DualQuant paper
rests on, Figure 2 (b)); here each is checked against an exhaustive scan of the admissible
values, and every vectorised sum against a pure-Python loop over the elements.
"""
import itertools

import numpy as np
import pytest

from oracle import formats as F
from oracle import solver as S

KINDS = ["INT4", "MXINT4", "MXFP4", "NVFP4", "INT8", "MXINT8"]
M, N, B = 4, 8, 4


def _grid(fmt):
    if fmt.elem in ("int4", "int8"):
        return np.arange(-fmt.qmax, fmt.qmax + 1, dtype=np.float64)
    return np.concatenate([-F.E2M1_MAG[:0:-1], F.E2M1_MAG])


def _admissible(fmt, s_t):
    """Every value of the block-scale set S (bf16: every positive normal finite value)."""
    if fmt.scale == "e8m0":
        return 2.0 ** np.arange(-127, 128)
    if fmt.scale == "e4m3":
        return (np.float32(s_t) * F.E4M3_POS[1:].astype(np.float32)).astype(np.float64)
    bits = np.arange(0x0080, 0x7F80, dtype=np.uint32)
    return (bits << 16).view(np.float32).astype(np.float64)


def _case(kind, seed):
    rng = np.random.default_rng(seed)
    fmt = F.make_format(kind, B)
    W = rng.standard_normal((M, N)).astype(np.float32).astype(np.float64) * 0.02
    W[0, 1] = 0.0
    s_t = S.tensor_scale(W, fmt)
    grid = _grid(fmt)
    q = rng.choice(grid[grid != 0], (M, N))
    q[1, 2] = 0.0
    c = rng.uniform(0.5, 2.0, N).astype(np.float32)
    return fmt, W, s_t, q, c


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("seed", range(6))
def test_r_step_is_exact_block_minimiser(kind, seed):
    fmt, W, s_t, q, c = _case(kind, seed)
    r_old = np.ones((M, N // B), dtype=np.float32)
    codes_old = np.zeros((M, N // B), dtype=np.uint16)
    _, r_new, num, den = S.r_step(W, q, c, r_old, codes_old, fmt, s_t)
    cand = _admissible(fmt, s_t)
    for i, b in itertools.product(range(M), range(N // B)):
        # pure-Python sums over the block
        nm = sum(W[i, j] * q[i, j] * float(c[j]) for j in range(b * B, (b + 1) * B))
        dn = sum((q[i, j] * float(c[j])) ** 2 for j in range(b * B, (b + 1) * B))
        assert num[i, b] == pytest.approx(nm, rel=1e-13, abs=1e-300)
        assert den[i, b] == pytest.approx(dn, rel=1e-13)

        def f(rv):
            cols = slice(b * B, (b + 1) * B)
            return np.sum((W[i, cols][None, :] - np.asarray(rv)[:, None] * q[i, cols][None, :]
                           * c[cols].astype(np.float64)[None, :]) ** 2, axis=1)
        # unprojected closed form beats a dense scan around it
        rstar = nm / dn
        scan = np.linspace(0.5 * rstar, 1.5 * rstar, 10001)
        assert f([rstar])[0] <= f(scan).min() * (1 + 1e-12) + 1e-300
        # projected value is the best admissible value (up to the binary32 rounding of r*)
        fbest = f(cand).min()
        assert f([float(r_new[i, b])])[0] <= fbest * (1 + 1e-6) + 1e-30


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("seed", range(6))
def test_c_step_is_exact_column_minimiser(kind, seed):
    fmt, W, s_t, q, _ = _case(kind, seed)
    rng = np.random.default_rng(100 + seed)
    r = rng.choice(_admissible(fmt, s_t)[-40:-20] if fmt.scale == "e4m3" else
                   2.0 ** np.arange(-8, -3), (M, N // B)).astype(np.float32)
    c_old = np.full(N, 3.0, dtype=np.float32)
    c_new, Nj, Dj = S.c_step(W, q, r, c_old, B)
    for j in range(N):
        nn = sum(W[i, j] * q[i, j] * float(r[i, j // B]) for i in range(M))
        dd = sum((q[i, j] * float(r[i, j // B])) ** 2 for i in range(M))
        assert Nj[j] == pytest.approx(nn, rel=1e-13, abs=1e-300)
        assert Dj[j] == pytest.approx(dd, rel=1e-13)

        def g(cv):
            return np.sum((W[:, j][None, :] - np.asarray(cv)[:, None] *
                           (q[:, j] * r[:, j // B].astype(np.float64))[None, :]) ** 2, axis=1)
        if dd > 0:
            cstar = nn / dd
            scan = np.linspace(cstar - abs(cstar), cstar + abs(cstar), 10001)
            assert g([float(c_new[j])])[0] <= g(scan).min() * (1 + 1e-9) + 1e-300
            assert c_new[j] == np.float32(cstar)
        else:
            assert c_new[j] == c_old[j]


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("seed", range(4))
def test_q_step_picks_nearest_grid_point(kind, seed):
    fmt = F.make_format(kind, B)
    rng = np.random.default_rng(200 + seed)
    W = (rng.standard_normal((M, N)) * 0.02).astype(np.float32).astype(np.float64)
    s_t = S.tensor_scale(W, fmt)
    _, r = S.init_scales(W, fmt, s_t)
    c = rng.uniform(0.5, 2.0, N).astype(np.float32)
    _, q, _ = S.q_step(W, r, c, fmt)
    grid = _grid(fmt)
    for i, j in itertools.product(range(M), range(N)):
        scale = float(r[i, j // B]) * float(c[j])
        errs = (W[i, j] - scale * grid) ** 2
        best = grid[np.argmin(errs)]
        if q[i, j] != best:
            # only allowed where the exact quotient sits on a rounding midpoint up to
            # the binary32 rounding of the quotient
            x = W[i, j] / scale
            mids = (grid[:-1] + grid[1:]) / 2
            assert np.min(np.abs(mids - x)) <= 1e-6 * max(abs(x), 1.0)
            assert abs(errs[np.searchsorted(grid, q[i, j])] - errs.min()) <= 1e-9 * W[i, j] ** 2


@pytest.mark.parametrize("kind", KINDS)
def test_mse_matches_elementwise_loop(kind):
    fmt, W, s_t, q, c = _case(kind, 7)
    r = np.full((M, N // B), 0.004, dtype=np.float32)
    got = S.mse(W, q, r, c, B)
    num = 0.0
    den = 0.0
    for i, j in itertools.product(range(M), range(N)):
        e = W[i, j] - float(r[i, j // B]) * q[i, j] * float(c[j])
        num += e * e
        den += W[i, j] ** 2
    assert got == pytest.approx(num / den, rel=1e-12)


@pytest.mark.parametrize("kind", KINDS)
def test_init_is_absmax_over_qmax_projected(kind):
    fmt = F.make_format(kind, B)
    rng = np.random.default_rng(9)
    W = (rng.standard_normal((M, N)) * 0.02).astype(np.float32).astype(np.float64)
    W[2, 4:8] = 0.0                                     # an all-zero block
    s_t = S.tensor_scale(W, fmt)
    _, r = S.init_scales(W, fmt, s_t)
    cand = _admissible(fmt, s_t)
    for i, b in itertools.product(range(M), range(N // B)):
        a = max(abs(W[i, j]) for j in range(b * B, (b + 1) * B))
        target = np.float32(a) / np.float32(fmt.qmax) if a > 0 else 1.0
        d = np.abs(cand - float(target))
        assert abs(float(r[i, b]) - float(target)) <= d.min() * (1 + 1e-6) + 1e-30
