"""Row-only / column-only updates and the Q-change trace on the GPU (B200).

The ablation of the ai4snews summary of DualQuant (paragraph 2: only the row or only the
column scales) and the relative change of Q-hat of Figure 2 (a) of the DualQuant paper,
through dq_solve_batched_ex. Checked: parity with the oracle's modes; the kept scale never
moves; the trace requested alongside changes no other output bit; the trace equals the
definition applied to the GPU's own Q of consecutive iterations (solves stopped after t-1
and t iterations), bit for bit; and it tracks the oracle's trace.
"""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import solver as S
from tests._parity import (compare_solve, assert_monotone, oracle_format, oracle_solve,
                           to_host, torch_to_f64)

pytestmark = pytest.mark.gpu

FMTS = ["INT4", "MXINT4", "MXFP4", "NVFP4", "INT8", "MXINT8"]


@pytest.fixture(scope="module")
def dq():
    import calibration_free_dual_b200 as pkg
    return pkg


def _matrix(seed, m, n):
    rng = np.random.default_rng(seed)
    w = rng.standard_t(4, (m, n)) * 0.014
    w[:, rng.choice(n, 3, replace=False)] *= 10.0
    return torch.from_numpy(w.astype(np.float32)).to(torch.bfloat16)


def _solve(dq, W, fmt_name, iters, **kw):
    out = dq.solve_batched([W.cuda()], fmt_name, iters, **kw)[0]
    torch.cuda.synchronize()
    assert dq.last_device_error() == 0
    h = to_host(out)
    if "qchange" in out:
        h["qchange"] = out["qchange"].cpu().numpy()
    return h


@pytest.mark.parametrize("fmt_name", FMTS)
@pytest.mark.parametrize("update", ["row", "col"])
def test_single_side_update_matches_oracle(dq, fmt_name, update):
    W = _matrix(77, 384, 512)
    fmt = oracle_format(fmt_name)
    h = _solve(dq, W, fmt_name, 10, update=update)
    h_prev = _solve(dq, W, fmt_name, 9, update=update)
    Wd = torch_to_f64(W)
    ora = oracle_solve(Wd, fmt, 10, update=update)
    compare_solve(h, ora, fmt, W=Wd, h_prev=h_prev, update=update, label=f"{fmt_name}/{update}")
    assert_monotone(h["mse"], label=f"{fmt_name}/{update}")
    if update == "row":
        np.testing.assert_array_equal(h["c"], np.ones(512, np.float32))
    else:
        r_init = to_host(dq.solve_batched([W.cuda()], fmt_name, 0)[0])["r"]
        np.testing.assert_array_equal(h["r"], r_init)


@pytest.mark.parametrize("fmt_name", FMTS)
def test_qchange_request_changes_nothing_else(dq, fmt_name):
    W = _matrix(78, 640, 256)
    plain = _solve(dq, W, fmt_name, 8)
    traced = _solve(dq, W, fmt_name, 8, qchange=True)
    for key in ("q_packed", "r", "c", "block_scales", "mse", "tensor_scale"):
        np.testing.assert_array_equal(traced[key], plain[key], err_msg=key)


@pytest.mark.parametrize("fmt_name", ["MXFP4", "NVFP4", "INT4", "MXINT8"])
@pytest.mark.parametrize("update", ["both", "row"])
def test_qchange_is_the_definition_on_the_gpus_own_q(dq, fmt_name, update):
    """A solve stopped after t iterations returns Q^t, so the trace of one long solve must
    equal ||Q^t - Q^(t-1)|| / ||Q^(t-1)|| formed from solves of t-1 and t iterations."""
    W = _matrix(79, 300, 256)
    fmt = oracle_format(fmt_name)
    T = 7
    h = _solve(dq, W, fmt_name, T, update=update, qchange=True)
    qc = h["qchange"]
    assert qc[0] == 0.0 and qc[1] == 0.0
    qs = []
    for t in range(T + 1):
        ht = _solve(dq, W, fmt_name, t, update=update)
        qs.append(F.decode_elem(F.unpack_codes(ht["q_packed"], fmt.bits), fmt).astype(np.float64))
    for t in range(2, T + 1):
        den = np.sqrt(np.sum(qs[t - 1] ** 2))
        want = np.sqrt(np.sum((qs[t] - qs[t - 1]) ** 2)) / den if den > 0 else 0.0
        assert qc[t] == want, (t, qc[t], want)


@pytest.mark.parametrize("fmt_name", FMTS)
def test_qchange_tracks_the_oracle(dq, fmt_name):
    W = _matrix(80, 512, 512)
    fmt = oracle_format(fmt_name)
    h = _solve(dq, W, fmt_name, 12, qchange=True)
    ora = S.solve(W.float().numpy().astype(np.float64), fmt, 12)
    scale = max(float(ora["qchange"].max()), 1e-12)
    np.testing.assert_allclose(h["qchange"], ora["qchange"], rtol=0.05, atol=0.02 * scale)


def test_bad_update_mode_is_rejected(dq):
    import ctypes
    W = _matrix(1, 16, 32).cuda()
    o = dq.api.solve_outputs(16, 32, dq.fmt_of("MXFP4"), 2, W.device)
    mats = (dq.dq_matrix * 1)()
    mats[0] = dq.dq_matrix(W.data_ptr(), 16, 32, 32, None, None, o["q_packed"].data_ptr(),
                           o["r"].data_ptr(), o["c"].data_ptr(), o["block_scales"].data_ptr(),
                           o["tensor_scale"].data_ptr(), o["mse"].data_ptr())
    opts = dq.dq_solve_options(7, None)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=W.device)
    st = dq.dq_solve_batched_ex(mats, 1, dq.DQ_BF16, dq.fmt_of("MXFP4"), 2, ctypes.byref(opts),
                                ctypes.c_void_p(ws.data_ptr()), ws.numel(), None)
    assert st == 1                                   # DQ_ERR_INVALID_ARG, nothing queued
