"""Pins of the SINQ-style baseline (oracle/sinq.py), the comparison of the DualQuant page's
Figure 1 (c): single-scale RTN vs SINQ's imbalance-minimising row/column normalisation vs
the dual-scale solve. The imbalance and the normalisation are pinned by hand values and
invariants; the ratios on the 512 x 512 tile are a reported measurement (the figure's tile
is not printed), checked only for the order the figure shows."""
import numpy as np
import pytest

from oracle import formats as F
from oracle import sinq as Q
from oracle import solver as S


def _circulant(v):
    v = np.asarray(v, dtype=np.float64)
    return np.stack([np.roll(v, k) for k in range(len(v))])


def test_imbalance_hand_values():
    # rows: std 1/2 and 1; columns: 1 and 3/2 (population deviations) -> 3/2 / 1/2 = 3
    assert Q.imbalance(np.array([[1.0, 2.0], [3.0, 5.0]])) == pytest.approx(3.0, rel=1e-15)
    # a circulant matrix of a zero-mean vector: every row and column the same multiset
    assert Q.imbalance(_circulant([1.0, -1.0, 2.0, -2.0, 0.5, -0.5])) == pytest.approx(1.0,
                                                                                     rel=1e-15)
    # a constant column has deviation 0: unbounded imbalance
    assert Q.imbalance(np.array([[0.0, 2.0], [0.0, 4.0]])) == float("inf")


def test_imbalance_invariances():
    rng = np.random.default_rng(3)
    W = rng.standard_t(4, (24, 40))
    i0 = Q.imbalance(W)
    assert Q.imbalance(7.5 * W) == pytest.approx(i0, rel=1e-14)
    assert Q.imbalance(-W) == pytest.approx(i0, rel=1e-14)
    assert Q.imbalance(W[rng.permutation(24)][:, rng.permutation(40)]) == pytest.approx(
        i0, rel=1e-14)
    assert Q.imbalance(W.T) == pytest.approx(i0, rel=1e-14)


def test_normalisation_recovers_a_scaled_balanced_matrix():
    """W = diag(a) C diag(b) with C balanced: the alternating normalisation reaches
    imbalance 1 and W = diag(s) W' diag(t) holds exactly."""
    rng = np.random.default_rng(4)
    C = _circulant(rng.standard_normal(32) - 0.0)
    C = C - C.mean()                                 # rows and columns zero-mean alike
    a = np.exp(rng.normal(0, 1.0, 32))
    b = np.exp(rng.normal(0, 1.0, 32))
    W = a[:, None] * C * b[None, :]
    s, t, Wn = Q.normalise(W, 24)
    assert Q.imbalance(W) > 5.0
    assert Q.imbalance(Wn) < 1.0 + 1e-6
    np.testing.assert_allclose(s[:, None] * Wn * t[None, :], W, rtol=1e-12)


def test_normalisation_commutes_with_permutations():
    rng = np.random.default_rng(5)
    W = rng.standard_t(4, (16, 32))
    W[:, 3] *= 20.0
    pr, pc = rng.permutation(16), rng.permutation(32)
    s, t, Wn = Q.normalise(W, 10)
    s2, t2, Wn2 = Q.normalise(W[pr][:, pc], 10)
    np.testing.assert_allclose(s2, s[pr], rtol=1e-12)
    np.testing.assert_allclose(t2, t[pc], rtol=1e-12)
    np.testing.assert_allclose(Wn2, Wn[pr][:, pc], rtol=1e-12)


def test_sinq_on_a_balanced_matrix_is_single_scale():
    """A matrix SINQ cannot improve (already balanced, uniform deviations) keeps s = t = 1:
    its reconstruction is plain single-scale RTN."""
    C = _circulant([1.0, -1.0, 2.0, -2.0] * 8)
    fmt = F.make_format("INT4", 32)
    What, imb = Q.sinq_reconstruct(C, fmt, 8)
    rtn = S.solve(C, fmt, 0)
    np.testing.assert_array_equal(What, S.reconstruct(rtn["q"], rtn["r"], rtn["c"], 32))
    assert imb == pytest.approx(1.0, rel=1e-12)


@pytest.mark.parametrize("kind,group", [("INT4", 128), ("MXFP4", 32)])
def test_dual_scale_beats_sinq_beats_single_on_the_512_tile(kind, group):
    import workloads as wl
    cfg = wl.CONFIGS[1]
    W = wl.weight_host(cfg, 0, 0).numpy().astype(np.float64)
    r = Q.mse_ratios(W, F.make_format(kind, group), cfg.iters)
    assert r["ratio_dual"] > r["ratio_sinq"] > 1.0, r
    assert r["imbalance_sinq"] < r["imbalance_dual"], r      # low imbalance, higher error
