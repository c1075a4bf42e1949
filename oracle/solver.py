"""Dual-scale BCD weight-reconstruction solver (oracle; test only).

Follows the DualQuant pages: the abstract of "DualQuant: Dual-scale Calibration-free
Weight-and-Activation Quantization for LLMs" (weight-reconstruction MSE, variable
splitting, block coordinate descent with a closed-form update for every block), the
acceptodds.com abstract (quantizer as a black box, scales projected onto the format's
admissible set after each update) and the ai4snews summary (a row scale and a column scale
per matrix). Figure 2 / Figure 3 of the first page give the two traces recorded here
(normalised MSE, monotone by Theorem 1 (i); relative change of Q-hat).

Model: W_hat[i, j] = r[i, j // B] * q[i, j] * c[j]. One iteration runs, in this order,
  Q-step  q = RNE_E( fl32( fl32(W * fl32(1/c)) * fl32(1/r) ) )
  r-step  r = Pi_S( fl32( sum_b W q c / sum_b (q c)^2 ) )       (kept where the sum is 0)
  c-step  c = fl32( sum_i W q r / sum_i (q r)^2 )               (kept where the sum is 0)
Sums and the traces are binary64; the code decisions are taken on binary32 values.

Ablation modes (the ai4snews summary, paragraph 2: turning on only the row scales or only
the column scales): update="row" runs the Q- and r-steps only (c stays at its initial value),
update="col" the Q- and c-steps only (r stays at its initial projected value). Each kept step
is still an exact block minimiser, so the trace stays monotone.
"""
from __future__ import annotations

import numpy as np

from .formats import (Format, round_elem, project_scale, nvfp4_tensor_scale)


def _blocks(a: np.ndarray, B: int) -> np.ndarray:
    """View [m, n] as [m, n/B, B] (blocks of B contiguous columns of one row)."""
    m, n = a.shape
    return a.reshape(m, n // B, B)


def _expand(r: np.ndarray, B: int) -> np.ndarray:
    """Row-block scales [m, n/B] -> per-element [m, n]."""
    return np.repeat(r, B, axis=1)


def tensor_scale(W: np.ndarray, fmt: Format, amax: float | None = None):
    """NVFP4 per-tensor scale s_t = fl32(amax|W| / 2688); None for the other formats.

    `amax` overrides the matrix's own amax (used when solving one column strip of a larger
    matrix, whose tensor scale comes from the whole matrix)."""
    if fmt.kind != "NVFP4":
        return None
    a = float(np.max(np.abs(W))) if amax is None else float(amax)
    return nvfp4_tensor_scale(a)


def init_scales(W: np.ndarray, fmt: Format, s_t=None):
    """Iteration-0 row-block scales: Pi_S(fl32(absmax / q_max)), Pi_S(1) for a zero block."""
    B = fmt.block
    a = np.max(np.abs(_blocks(W, B)), axis=2)                       # [m, n/B], exact
    v = (a.astype(np.float32) / np.float32(fmt.qmax)).astype(np.float32)
    v = np.where(a > 0, v, np.float32(1.0)).astype(np.float32)
    codes, r = project_scale(v, fmt, s_t)
    return codes, r


def q_step(W: np.ndarray, r: np.ndarray, c: np.ndarray, fmt: Format):
    """Black-box quantizer: codes of diag(1/r) W diag(1/c) on the element grid.

    Returns (codes uint8 [m, n], q float64 [m, n], x binary32 [m, n])."""
    W32 = W.astype(np.float32)
    ic = (np.float32(1.0) / c.astype(np.float32)).astype(np.float32)          # [n]
    ir = (np.float32(1.0) / r.astype(np.float32)).astype(np.float32)          # [m, n/B]
    y = (W32 * ic[None, :]).astype(np.float32)
    x = (y * _expand(ir, fmt.block)).astype(np.float32)
    codes, q = round_elem(x, fmt)
    return codes, q, x


def r_step_unprojected(W: np.ndarray, q: np.ndarray, c: np.ndarray, B: int):
    """num, den of the least-squares row-block scale given (q, c), binary64."""
    qc = q * c.astype(np.float64)[None, :]
    num = np.sum(_blocks(W * qc, B), axis=2)
    den = np.sum(_blocks(qc * qc, B), axis=2)
    return num, den


def r_step(W, q, c, r_old, r_codes_old, fmt: Format, s_t=None):
    """Closed-form r given (q, c), projected onto the admissible set; kept where den = 0."""
    num, den = r_step_unprojected(W, q, c, fmt.block)
    ok = den > 0
    with np.errstate(divide="ignore", invalid="ignore"):
        rstar = np.where(ok, num / np.where(ok, den, 1.0), 1.0).astype(np.float32)
    codes, r = project_scale(rstar, fmt, s_t)
    r = np.where(ok, r, r_old).astype(np.float32)
    codes = np.where(ok, codes, r_codes_old).astype(r_codes_old.dtype)
    return codes, r, num, den


def c_step_sums(W: np.ndarray, q: np.ndarray, r: np.ndarray, B: int):
    """N_j = sum_i W q r and D_j = sum_i (q r)^2 per column, binary64."""
    qr = q * _expand(r.astype(np.float64), B)
    return np.sum(W * qr, axis=0), np.sum(qr * qr, axis=0)


def c_step(W, q, r, c_old, B: int):
    """Closed-form column scale given (q, r); kept where D = 0. Not projected."""
    N, D = c_step_sums(W, q, r, B)
    ok = D > 0
    with np.errstate(divide="ignore", invalid="ignore"):
        c = np.where(ok, (N / np.where(ok, D, 1.0)), c_old).astype(np.float32)
    return c, N, D


def reconstruct(q: np.ndarray, r: np.ndarray, c: np.ndarray, B: int) -> np.ndarray:
    return _expand(r.astype(np.float64), B) * q * c.astype(np.float64)[None, :]


def mse(W: np.ndarray, q: np.ndarray, r: np.ndarray, c: np.ndarray, B: int) -> float:
    """Normalised reconstruction error ||W - W_hat||_F^2 / ||W||_F^2 (0 for W = 0)."""
    wsq = float(np.sum(W * W))
    if wsq == 0.0:
        return 0.0
    e = W - reconstruct(q, r, c, B)
    return float(np.sum(e * e)) / wsq


UPDATES = ("both", "row", "col")


def solve(W, fmt: Format, iters: int, r0=None, c0=None, amax=None, keep_history=False,
          update: str = "both"):
    """Run the dual-scale BCD solve of one matrix.

    W: [m, n] array of binary32-representable values (bf16 or fp32 weights).
    r0 / c0: optional warm start (r0 is projected; c0 must be finite and positive).
    amax: NVFP4 only, overrides the matrix amax for the tensor scale.
    update: "both" (the method), "row" (r only) or "col" (c only).
    Returns a dict with q (values), codes, r, r_codes, c, s_t, mse [T+1], qchange [T+1]
    and, with keep_history, the states (r, c) before each iteration's Q-step.
    """
    if update not in UPDATES:
        raise ValueError("update must be one of %s" % (UPDATES,))
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    B = fmt.block
    if n % B:
        raise ValueError("n must be a multiple of the block length")
    s_t = tensor_scale(W, fmt, amax)
    if c0 is None:
        c = np.ones(n, dtype=np.float32)
    else:
        c = np.asarray(c0, dtype=np.float32).copy()
        if not (np.all(np.isfinite(c)) and np.all(c > 0)):
            raise ValueError("c0 must be finite and positive")
    if r0 is None:
        r_codes, r = init_scales(W, fmt, s_t)
    else:
        r_codes, r = project_scale(np.asarray(r0, dtype=np.float32), fmt, s_t)
    codes, q, _ = q_step(W, r, c, fmt)
    trace = [mse(W, q, r, c, B)]
    qchange = [0.0]
    history = []
    for _ in range(iters):
        if keep_history:
            history.append((r.copy(), c.copy(), r_codes.copy()))
        q_prev = q
        codes, q, _ = q_step(W, r, c, fmt)
        if update != "col":
            r_codes, r, _, _ = r_step(W, q, c, r, r_codes, fmt, s_t)
        if update != "row":
            c, _, _ = c_step(W, q, r, c, B)
        trace.append(mse(W, q, r, c, B))
        nprev = float(np.linalg.norm(q_prev))
        qchange.append(float(np.linalg.norm(q - q_prev)) / nprev if nprev > 0 else 0.0)
    out = dict(q=q, codes=codes, r=r, r_codes=r_codes, c=c, s_t=s_t,
               mse=np.array(trace), qchange=np.array(qchange))
    if keep_history:
        out["history"] = history
    return out
