"""SINQ-style dual-scale baseline: matrix imbalance and alternating row/column normalisation
(oracle, test infrastructure only).

The DualQuant page's Figure 1 compares scale designs on one weight tile: single-scale RTN;
SINQ, whose objective is the matrix imbalance (it reaches 1.65 there, with 3.32 times less
MSE than single-scale); and DualQuant's MSE-driven solve (12.54 times less). The pages name
the imbalance as SINQ's objective without defining it. The reading used here (from the SINQ method's public description): the
imbalance of W is the largest over the smallest of all row and column standard
deviations,
    I(W) = max(sigma_rows, sigma_cols) / min(sigma_rows, sigma_cols),
and SINQ lowers it by alternately dividing every row and every column by its standard
deviation (a Sinkhorn-Knopp-style iteration on the standard deviations), accumulating the
row scales s and column scales t and keeping the iterate of lowest imbalance. The
normalised matrix W' = diag(1/s) W diag(1/t) is then quantized by single-scale RTN in the
target format, and W_hat = diag(s) RTN(W') diag(t).

Only used to place the 512 x 512 tile's dual/single MSE ratio next to the figure's; the
figure's tile values are not printed, so its numbers are context, not a target.
"""
from __future__ import annotations

import numpy as np

from . import solver as S
from .formats import Format


def imbalance(W: np.ndarray) -> float:
    """Largest over smallest standard deviation across all rows and columns of W."""
    W = np.asarray(W, dtype=np.float64)
    sd = np.concatenate([W.std(axis=1), W.std(axis=0)])
    lo = float(sd.min())
    return float("inf") if lo == 0.0 else float(sd.max()) / lo


def normalise(W: np.ndarray, iters: int = 16):
    """Alternating row / column standard-deviation normalisation.

    Returns (s, t, W') with W = diag(s) W' diag(t), for the iterate of lowest imbalance
    (iterate 0 is W itself with s = t = 1). Rows or columns with zero deviation keep their
    scale."""
    W = np.asarray(W, dtype=np.float64)
    s = np.ones(W.shape[0])
    t = np.ones(W.shape[1])
    cur = W.copy()
    best = (imbalance(cur), s.copy(), t.copy(), cur.copy())
    for _ in range(iters):
        sr = cur.std(axis=1)
        sr = np.where(sr > 0, sr, 1.0)
        cur = cur / sr[:, None]
        s = s * sr
        sc = cur.std(axis=0)
        sc = np.where(sc > 0, sc, 1.0)
        cur = cur / sc[None, :]
        t = t * sc
        imb = imbalance(cur)
        if imb < best[0]:
            best = (imb, s.copy(), t.copy(), cur.copy())
    _, s, t, cur = best
    return s, t, cur


def sinq_reconstruct(W: np.ndarray, fmt: Format, iters: int = 16):
    """(W_hat, imbalance of the normalised matrix): SINQ's normalisation, then single-scale
    RTN of the normalised matrix in `fmt` (the iteration-0 state of the dual-scale solve,
    i.e. c = 1 and block scales Pi_S(absmax / q_max)), then the scales put back."""
    s, t, Wn = normalise(W, iters)
    Wn32 = Wn.astype(np.float32).astype(np.float64)
    out = S.solve(Wn32, fmt, 0)
    rec = S.reconstruct(out["q"], out["r"], out["c"], fmt.block)
    return s[:, None] * rec * t[None, :], imbalance(Wn32)


def mse_ratios(W: np.ndarray, fmt: Format, dual_iters: int, sinq_iters: int = 16) -> dict:
    """Single-scale MSE over SINQ's and over the dual-scale solve's, on one matrix."""
    W = np.asarray(W, dtype=np.float64)
    wsq = float(np.sum(W * W))
    single = S.solve(W, fmt, 0)["mse"][0]
    What, imb = sinq_reconstruct(W, fmt, sinq_iters)
    sinq = float(np.sum((W - What) ** 2)) / wsq
    dual = S.solve(W, fmt, dual_iters)
    return {"mse_single": float(single), "mse_sinq": sinq, "mse_dual": float(dual["mse"][-1]),
            "ratio_sinq": float(single) / sinq, "ratio_dual": float(single / dual["mse"][-1]),
            "imbalance_W": imbalance(W), "imbalance_sinq": imb,
            # the matrix the dual-scale quantizer rounds: W / (r c)
            "imbalance_dual": imbalance(W / (dual["r"].astype(np.float64).repeat(fmt.block, axis=1)
                                             * dual["c"].astype(np.float64)[None, :]))}


if __name__ == "__main__":      # the 512 x 512 fp32 INT4 g=128 tile's figures
    import json
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import workloads as wl
    from .formats import make_format
    cfg = wl.CONFIGS[1]
    W = wl.weight_host(cfg, 0, 0).numpy().astype(np.float64)
    print(json.dumps(mse_ratios(W, make_format("INT4", 128), cfg.iters), indent=1))
