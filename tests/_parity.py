"""Comparison of CUDA-path outputs with the oracle (test helper, not collected).

The bar has two parts.

1. Every BCD step of the GPU's own last iteration, replayed by the oracle's step functions
   from the GPU's own state (`h_prev`: the same solve stopped one iteration earlier, whose
   outputs are the state the last iteration started from):
     * Q-step: the GPU's codes equal the oracle's Q-step on (r, c) of `h_prev`, everywhere
       (the decision is taken on the same binary32 quotient on both sides);
     * r-step + projection: every block-scale code equals Pi_S of the binary64 least-squares
       quotient formed from the GPU's own (q, c_prev), except where that quotient lies within
       PROJ_REL of the boundary between the two candidates (the GPU's block sums are
       binary32 for the E4M3 and E8M0 formats); an empty block keeps its previous code;
     * c-step: every c_j is within C_STEP_REL of fl32(N_j / D_j) formed in binary64 from the
       GPU's own (q, r);
     * trace: the last MSE entry is within the MSE bar of the MSE of the GPU's own final state
       computed directly in binary64.
2. The GPU trajectory against the oracle's (the same seeded input):
     * element codes: >= 99.9% identical; at every mismatch either the element's block scale
       differed in the state of the last Q-step, or the two sides' binary32 quotients lie on
       the two sides of (or on) the rounding midpoint between the two codes: a decision at a
       rounding boundary, moved by the last bits of c;
     * block scales: >= 99.9% identical, mismatches one admissible step apart, each with the
       two sides' least-squares quotients on the two sides of the projection boundary (within
       PROJ_REL), or in a row block whose element codes differ; blocks with equal codes have
       bit-identical decoded r;
     * ||c_gpu - c_ora|| / ||c_ora|| <= 1e-4;
     * normalised MSE at every iteration: |mse_gpu - mse_ora| <= 1e-4 * mse_ora for the 4-bit
       formats (no absolute floor). The 8-bit formats (MSE 1e-5..1e-4) add MSE_ABS_8BIT =
       1e-7: the GPU forms the trace from the expansion ||W||^2 - 2 sum c_j N_j + sum c_j^2 D_j
       with binary32 partial sums, whose three terms are each about ||W||^2, so its absolute
       error in normalised units is a few 1e-8 (measured at most 2e-8) whatever the MSE;
     * NVFP4 tensor scale: bit-exact.
The measured agreement figures (code and scale match, ||dr||/||r||, c_rel, the largest MSE
deviation, the mismatch counts by explanation) are returned and collected in REPORTS; with
DQ_PARITY_REPORT set, the session writes them to that JSON file.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import formats as F
from oracle import solver as S

CODE_MATCH = 0.999
SCALE_MATCH = 0.999
C_REL = 1e-4
C_STEP_REL = 1e-5
MSE_REL = 1e-4
MSE_ABS_8BIT = 1e-7
PROJ_REL = 1e-5

REPORTS: list = []


def oracle_format(name_or_spec):
    if isinstance(name_or_spec, str):
        kind, group = {"INT4": ("INT4", 128), "INT4_G64": ("INT4", 64),
                       "MXINT4": ("MXINT4", 32), "MXFP4": ("MXFP4", 32),
                       "NVFP4": ("NVFP4", 16), "INT8": ("INT8", 128),
                       "INT8_G64": ("INT8", 64), "MXINT8": ("MXINT8", 32)}[name_or_spec]
    else:
        kind, group = name_or_spec.kind, name_or_spec.group
    return F.make_format(kind, group)


def to_host(out: dict) -> dict:
    h = {}
    for k, v in out.items():
        if k.startswith("_"):
            continue
        h[k] = v.detach().cpu().numpy()
    return h


def grid_index(q: np.ndarray, fmt) -> np.ndarray:
    """Position of each element value on the signed grid (-0 and +0 coincide)."""
    if fmt.elem in ("int4", "int8"):
        return np.rint(q).astype(np.int64)
    mag = np.abs(q)
    idx = np.searchsorted(F.E2M1_MAG, mag)
    return np.where(q < 0, -idx, idx)


def scale_codes_gpu(h: dict, fmt) -> np.ndarray:
    bs = h["block_scales"]
    if fmt.scale == "bf16":
        return bs.view(np.uint16).astype(np.int64)
    return bs.astype(np.int64)


def _codes_values(h: dict, fmt):
    codes = F.unpack_codes(h["q_packed"], fmt.bits)
    return codes, F.decode_elem(codes, fmt)


def _decoded_scales(codes: np.ndarray, fmt, s_t) -> np.ndarray:
    return F.decode_scale(codes, fmt, s_t).astype(np.float64)


def _mse_ok(mg: np.ndarray, mo: np.ndarray, fmt) -> np.ndarray:
    bar = MSE_REL * np.abs(mo)
    if fmt.bits == 8:
        bar = bar + MSE_ABS_8BIT
    return np.abs(mg - mo) <= bar


def _straddle(a: np.ndarray, b: np.ndarray, mid: np.ndarray, rel: float) -> np.ndarray:
    """a and b lie on the two sides of mid (or on it), up to a relative slack."""
    lo, hi = np.minimum(a, b), np.maximum(a, b)
    return (lo <= mid * (1 + rel)) & (hi >= mid * (1 - rel))


def _check_own_steps(h, h_prev, W, fmt, s_t, update, label, rep, trace=True):
    """Part 1: the GPU's last iteration replayed from its own state by the oracle's steps."""
    B = fmt.block
    codes_g, qg = _codes_values(h, fmt)
    sc_g = scale_codes_gpu(h, fmt)
    sc_prev = scale_codes_gpu(h_prev, fmt)
    r_prev = h_prev["r"].astype(np.float32)
    c_prev = h_prev["c"].astype(np.float32)
    # Q-step
    codes_own, _, _ = S.q_step(W, r_prev, c_prev, fmt)
    bad_q = codes_own != codes_g
    assert not bad_q.any(), (label, "Q-step differs from the oracle's on the GPU's own state",
                             int(bad_q.sum()))
    # r-step and projection
    if update == "col":
        np.testing.assert_array_equal(sc_g, sc_prev, err_msg=label + ": r moved in col mode")
    else:
        num, den = S.r_step_unprojected(W, qg, c_prev, B)
        ok = den > 0
        with np.errstate(divide="ignore", invalid="ignore"):
            rstar = np.where(ok, num / np.where(ok, den, 1.0), 1.0)
        own_codes, _ = F.project_scale(rstar.astype(np.float32), fmt, s_t)
        own_codes = np.where(ok, own_codes.astype(np.int64), sc_prev)
        diff = own_codes != sc_g
        if diff.any():
            vg = _decoded_scales(sc_g[diff], fmt, s_t)
            vo = _decoded_scales(own_codes[diff], fmt, s_t)
            mid = 0.5 * (vg + vo)
            near = np.abs(rstar[diff] - mid) <= PROJ_REL * mid
            assert ok[diff].all() and near.all(), (
                label, "projection off the boundary", int((~near).sum()))
            assert np.all(np.abs(sc_g[diff] - own_codes[diff]) == 1), (label, "projection step")
        rep["own_scale_boundary"] = int(diff.sum())
    # c-step
    if update == "row":
        np.testing.assert_array_equal(h["c"], c_prev, err_msg=label + ": c moved in row mode")
    else:
        N, D = S.c_step_sums(W, qg, h["r"].astype(np.float32), B)
        okc = D > 0
        with np.errstate(divide="ignore", invalid="ignore"):
            c_own = np.where(okc, (N / np.where(okc, D, 1.0)).astype(np.float32), c_prev)
        rel = np.abs(h["c"].astype(np.float64) - c_own) / np.abs(c_own)
        rep["own_c_rel_max"] = float(rel.max()) if rel.size else 0.0
        assert rep["own_c_rel_max"] <= C_STEP_REL, (label, "c-step", rep["own_c_rel_max"])
    if not trace:
        return
    # trace, last entry, from the GPU's own final state
    m_own = S.mse(W, qg, h["r"].astype(np.float32), h["c"].astype(np.float32), B)
    assert _mse_ok(np.array([h["mse"][-1]]), np.array([m_own]), fmt).all(), (
        label, "final MSE against the GPU's own state", h["mse"][-1], m_own)


def compare_solve(h: dict, ora: dict, fmt, *, W: np.ndarray | None = None,
                  h_prev: dict | None = None, update: str = "both", exact: bool = False,
                  label: str = "", trace: bool = True) -> dict:
    """Assert the parity bar; return the measured agreement figures.

    h: GPU outputs (host arrays) after T iterations; ora: the oracle's solve of the same
    input (keep_history=True when T >= 1 and W is given); W: the input as binary64; h_prev:
    GPU outputs of the same solve stopped after T - 1 iterations (T >= 1); trace=False
    skips the MSE trace (outputs of a part of a matrix)."""
    T = len(h["mse"]) - 1
    s_t = ora.get("s_t")
    rep = dict(label=label, fmt=fmt.kind, block=fmt.block, iters=T)
    codes_g, qg = _codes_values(h, fmt)
    qo = ora["q"]
    same_q = grid_index(qg, fmt) == grid_index(qo, fmt)
    sc_g = scale_codes_gpu(h, fmt)
    sc_o = np.asarray(ora["r_codes"]).astype(np.int64)
    same_r = sc_g == sc_o
    rep["elements"] = int(same_q.size)
    rep["code_match"] = float(same_q.mean())
    rep["scale_match"] = float(same_r.mean())
    rg = h["r"].astype(np.float64)
    ro = np.asarray(ora["r"]).astype(np.float64)
    rep["r_rel"] = float(np.linalg.norm(rg - ro) / max(np.linalg.norm(ro), 1e-300))
    rep["c_rel"] = float(np.linalg.norm(h["c"].astype(np.float64) - ora["c"]) /
                         max(np.linalg.norm(ora["c"].astype(np.float64)), 1e-300))
    mo = np.asarray(ora["mse"])
    mg = h["mse"]
    rel = np.abs(mg - mo) / np.maximum(np.abs(mo), 1e-300)
    rel = np.where(mo == 0, np.abs(mg - mo), rel)
    rep["mse_rel_max"] = float(rel.max())
    rep["mse_abs_max"] = float(np.abs(mg - mo).max())
    if fmt.kind == "NVFP4" and "tensor_scale" in h:
        assert np.float32(h["tensor_scale"][0]) == np.float32(s_t), (label, "tensor scale")
    if exact:
        assert same_q.all(), (label, "codes differ", int((~same_q).sum()))
        assert same_r.all(), (label, "scales differ", int((~same_r).sum()))
    assert rep["code_match"] >= CODE_MATCH, (label, rep)
    assert rep["scale_match"] >= SCALE_MATCH, (label, rep)
    # blocks with equal codes decode to identical r
    blk_same = np.broadcast_to(same_r, rg.shape)
    assert np.array_equal(rg[blk_same], ro[blk_same]), (label, "r differs in matched blocks")
    # decoded r consistent with the codes (exactly)
    np.testing.assert_array_equal(h["r"], _decoded_scales(sc_g, fmt, s_t).astype(np.float32))
    assert np.all(np.abs(sc_g[~same_r] - sc_o[~same_r]) <= 1), (label, "scale step > 1")
    B = fmt.block
    if W is not None and T >= 1:
        assert h_prev is not None and "history" in ora, label
        _check_own_steps(h, h_prev, W, fmt, s_t, update, label, rep, trace)
        # code mismatches: block scale differed in the last Q-step's state, or the two
        # binary32 quotients straddle the midpoint between the two codes
        r_po, c_po, rc_po = ora["history"][T - 1]
        rc_pg = scale_codes_gpu(h_prev, fmt)
        blk_prev_diff = np.repeat(rc_pg != np.asarray(rc_po).astype(np.int64), B, axis=1)
        mis = ~same_q
        by_scale = mis & blk_prev_diff
        rest = mis & ~blk_prev_diff
        n_mid = 0
        if rest.any():
            _, _, xg = S.q_step(W, h_prev["r"].astype(np.float32),
                                h_prev["c"].astype(np.float32), fmt)
            _, _, xo = S.q_step(W, r_po, c_po, fmt)
            ag = np.abs(xg[rest].astype(np.float64))
            ao = np.abs(xo[rest].astype(np.float64))
            mid = 0.5 * (np.abs(qg[rest]) + np.abs(qo[rest]))
            steps = np.abs(grid_index(qg, fmt)[rest] - grid_index(qo, fmt)[rest])
            assert np.all(steps == 1), (label, "code mismatch beyond one step")
            strad = _straddle(ag, ao, mid, 0.0)
            assert strad.all(), (label, "code mismatch off a rounding midpoint",
                                 int((~strad).sum()))
            n_mid = int(rest.sum())
        rep["code_mis_by_scale"] = int(by_scale.sum())
        rep["code_mis_at_midpoint"] = n_mid
        # scale mismatches: the two sides' least-squares quotients straddle the boundary,
        # or the row block's codes differ
        if update != "col" and (~same_r).any():
            c_pg = h_prev["c"].astype(np.float32)
            ng, dg = S.r_step_unprojected(W, qg, c_pg, B)
            no, do = S.r_step_unprojected(W, qo, np.asarray(c_po, dtype=np.float32), B)
            codes_blk_diff = (~same_q).reshape(same_q.shape[0], -1, B).any(axis=2)
            m = ~same_r
            with np.errstate(divide="ignore", invalid="ignore"):
                rsg = ng[m] / dg[m]
                rso = no[m] / do[m]
            vg = _decoded_scales(sc_g[m], fmt, s_t)
            vo = _decoded_scales(sc_o[m], fmt, s_t)
            strad = _straddle(rsg, rso, 0.5 * (vg + vo), PROJ_REL)
            explained = strad | codes_blk_diff[m]
            assert explained.all(), (label, "scale mismatch off the projection boundary",
                                     int((~explained).sum()))
            rep["scale_mis_at_boundary"] = int(strad.sum())
            rep["scale_mis_by_codes"] = int((~strad & codes_blk_diff[m]).sum())
        else:
            rep["scale_mis_at_boundary"] = rep["scale_mis_by_codes"] = 0
    else:
        # no state to replay (iteration 0 only): mismatches one grid step, or in a block
        # whose scale differs
        blk_diff = np.repeat(~same_r, B, axis=1)
        step = np.abs(grid_index(qg, fmt) - grid_index(qo, fmt))
        bad = (~same_q) & (step > 1) & (~blk_diff)
        assert not bad.any(), (label, "code mismatches beyond one step", int(bad.sum()))
    assert rep["c_rel"] <= C_REL, (label, rep)
    if trace:
        assert _mse_ok(mg, mo, fmt).all(), (label, rep)
    REPORTS.append(rep)
    return rep


def gpu_pair(run, iters: int):
    """(outputs after `iters` iterations, outputs after iters - 1 or None): run(t) must solve
    the same input from the same start for t iterations and return host arrays."""
    h = run(iters)
    return h, (run(iters - 1) if iters >= 1 else None)


def oracle_solve(W: np.ndarray, fmt, iters: int, **kw) -> dict:
    return S.solve(W, fmt, iters, keep_history=True, **kw)


def assert_monotone(mse: np.ndarray, rel: float = 1e-6, label: str = "") -> None:
    assert np.all(mse[1:] <= mse[:-1] * (1 + rel)), (label, mse)


def torch_to_f64(W: torch.Tensor) -> np.ndarray:
    return W.detach().float().cpu().numpy().astype(np.float64)
