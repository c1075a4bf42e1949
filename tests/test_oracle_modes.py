"""Pins for the oracle's ablation modes and its Q-change trace (CPU only).

The ai4snews summary of DualQuant (paragraph 2) compares turning on only the row scales or
only the column scales with turning on both; Figure 2 (a) of the DualQuant paper plots the
relative change of Q-hat between BCD iterations. The pins below do not re-run the oracle's
own step functions: the row-only update is checked against a brute-force search over every
admissible scale value, the column-only update against the neighbouring binary32 values of
the 1-D quadratic it minimises, and the Q-change trace against invariants of its
definition.
"""
import numpy as np
import pytest

from oracle import formats as F
from oracle import solver as S

KINDS = ["INT4", "MXINT4", "MXFP4", "NVFP4", "INT8", "MXINT8"]


def _small(seed, m=24, n=64):
    rng = np.random.default_rng(seed)
    W = rng.standard_t(4, (m, n)) * 0.014
    W[:, rng.choice(n, 2, replace=False)] *= 8.0
    return W.astype(np.float32).astype(np.float64)


def _admissible(fmt, s_t):
    """Every admissible decoded block scale of the format (ascending, unique)."""
    if fmt.scale == "bf16":
        codes = np.arange(F.BF16_MIN_NORMAL_BITS, F.BF16_MAX_BITS + 1, dtype=np.uint16)
    elif fmt.scale == "e8m0":
        codes = np.arange(0, 255, dtype=np.int64)
    else:
        codes = np.arange(1, 127, dtype=np.int64)
    return np.unique(F.decode_scale(codes, fmt, s_t).astype(np.float64))


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("update", ["row", "col"])
def test_single_side_modes_keep_the_other_scale_and_stay_monotone(kind, update):
    fmt = F.make_format(kind)
    W = _small(3, 64, 256)
    out = S.solve(W, fmt, 12, update=update, keep_history=True)
    both = S.solve(W, fmt, 12)
    m = out["mse"]
    assert np.all(m[1:] <= m[:-1] * (1 + 1e-12)), m
    assert m[0] == both["mse"][0]
    r_init, c_init, codes_init = out["history"][0]
    if update == "row":
        np.testing.assert_array_equal(out["c"], np.ones(W.shape[1], np.float32))
    else:
        np.testing.assert_array_equal(out["r"], r_init)
        np.testing.assert_array_equal(out["r_codes"], codes_init)


@pytest.mark.parametrize("kind", KINDS)
def test_row_only_update_is_the_best_admissible_scale(kind):
    """One row-only iteration from RTN: each block's new scale minimises
    sum_b (W - r q c)^2 over all admissible values (q and c = 1 fixed)."""
    fmt = F.make_format(kind, {"INT4": 32, "MXINT4": 32, "MXFP4": 32, "NVFP4": 16, "INT8": 32,
                               "MXINT8": 32}[kind])
    W = _small(11, 6, 64)
    out = S.solve(W, fmt, 1, update="row")
    q, r = out["q"], out["r"].astype(np.float64)
    cand = _admissible(fmt, out["s_t"])
    B = fmt.block
    for i in range(W.shape[0]):
        for b in range(W.shape[1] // B):
            w = W[i, b * B:(b + 1) * B]
            qq = q[i, b * B:(b + 1) * B]
            if not np.any(qq):
                continue
            f = ((w[None, :] - cand[:, None] * qq[None, :]) ** 2).sum(axis=1)
            fr = ((w - r[i, b] * qq) ** 2).sum()
            assert fr <= f.min() * (1 + 1e-9) + 1e-300, (kind, i, b, fr, f.min())


@pytest.mark.parametrize("kind", KINDS)
def test_col_only_update_is_the_nearest_binary32_minimiser(kind):
    """One column-only iteration from RTN: each c_j is the binary32 value closest to the
    minimiser of sum_i (W_ij - r q_ij c)^2, so neither binary32 neighbour does better."""
    fmt = F.make_format(kind)
    W = _small(5, 40, 128)
    out = S.solve(W, fmt, 1, update="col")
    q, c = out["q"], out["c"]
    rb = np.repeat(out["r"].astype(np.float64), fmt.block, axis=1)
    for j in range(W.shape[1]):
        a = rb[:, j] * q[:, j]
        if not np.any(a):
            continue
        f = lambda cv: float(((W[:, j] - a * float(cv)) ** 2).sum())
        up = np.nextafter(c[j], np.float32(np.inf))
        dn = np.nextafter(c[j], np.float32(0))
        assert f(c[j]) <= min(f(up), f(dn)) * (1 + 1e-12), (kind, j)


@pytest.mark.parametrize("kind", KINDS)
def test_qchange_invariants(kind):
    """qchange[0] = qchange[1] = 0 (the first Q-step sees the initial state); the trace is
    unchanged by W -> -W (sign symmetry of the grids) and, for power-of-two block scales, by
    W -> 4W; it is zero along a fixed point."""
    fmt = F.make_format(kind)
    W = _small(9, 48, 256)
    out = S.solve(W, fmt, 10)
    qc = out["qchange"]
    assert qc.shape == (11,)
    assert qc[0] == 0.0 and qc[1] == 0.0
    assert np.all(qc >= 0) and np.any(qc[2:] > 0)
    np.testing.assert_array_equal(S.solve(-W, fmt, 10)["qchange"], qc)
    if fmt.scale == "e8m0":
        np.testing.assert_array_equal(S.solve(4.0 * W, fmt, 10)["qchange"], qc)
    # a fixed point: the reconstruction of a converged state, solved from that state
    fp = S.reconstruct(out["q"], out["r"], out["c"], fmt.block).astype(np.float32)
    fp = fp.astype(np.float64)
    again = S.solve(fp, fmt, 4, r0=out["r"], c0=out["c"],
                    amax=float(np.abs(W).max()) if kind == "NVFP4" else None)
    np.testing.assert_array_equal(again["qchange"], np.zeros(5))
