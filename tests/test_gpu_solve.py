"""Parity of the CUDA solve with the oracle on seeded inputs (B200).

Sizes span several column tiles, ragged last sweeps and tiles whose lower rows are re-read
from L2 on every pass, while the oracle still finishes in seconds. Tolerances are the ones written out in tests/_parity.py.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import solver as S
from tests._parity import (oracle_format, to_host, compare_solve, assert_monotone,
                           oracle_solve, torch_to_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dq():
    import calibration_free_dual_b200 as pkg
    return pkg


def _matrix(seed, m, n, dtype, dist="t4", outlier_cols=3):
    rng = np.random.default_rng(seed)
    if dist == "t4":
        w = rng.standard_t(4, (m, n)) * 0.014
    else:
        w = rng.standard_normal((m, n)) * 0.015
    if outlier_cols:
        w[:, rng.choice(n, min(outlier_cols, n), replace=False)] *= 10.0
    t = torch.from_numpy(w.astype(np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t


def _run(dq, Wt, fmt_name, iters, r0=None, c0=None):
    out = dq.solve(Wt.cuda(), fmt_name, iters,
                   r0=None if r0 is None else torch.from_numpy(r0).cuda(),
                   c0=None if c0 is None else torch.from_numpy(c0).cuda())
    torch.cuda.synchronize()
    assert dq.last_device_error() == 0
    return to_host(out)


def _check(dq, Wt, fmt_name, iters, label, r0=None, c0=None, **ora_kw):
    """GPU solve of T and T - 1 iterations against the oracle's solve with its history."""
    fmt = oracle_format(fmt_name)
    h = _run(dq, Wt, fmt_name, iters, r0=r0, c0=c0)
    h_prev = _run(dq, Wt, fmt_name, iters - 1, r0=r0, c0=c0) if iters >= 1 else None
    Wd = torch_to_f64(Wt)
    ora = oracle_solve(Wd, fmt, iters, r0=r0, c0=c0, **ora_kw)
    rep = compare_solve(h, ora, fmt, W=Wd, h_prev=h_prev, label=label)
    return h, ora, rep


CASES = [
    # fmt, dtype, m, n, iters
    ("INT4", "f32", 512, 512, 20),          # the 512x512 fp32 configuration's shape
    ("INT4", "bf16", 200, 384, 8),
    ("INT4_G64", "bf16", 130, 320, 8),
    ("INT4_G64", "f32", 67, 192, 6),
    ("MXINT4", "bf16", 257, 224, 8),
    ("MXINT4", "f32", 96, 160, 8),
    ("MXFP4", "bf16", 512, 2048, 16),       # 1B-shaped k_proj
    ("MXFP4", "f32", 33, 96, 8),
    ("NVFP4", "bf16", 640, 1040, 10),       # n = 65 blocks of 16: 16-column tiles
    ("NVFP4", "bf16", 1024, 1024, 16),
    ("NVFP4", "f32", 300, 512, 8),
    ("NVFP4", "bf16", 1, 64, 5),            # a single row
    ("MXFP4", "bf16", 2, 32, 5),            # one block column
    # the 8-bit formats (appendix 8-bit table): INT8 G=128/64 with bf16 scales, MXINT8 G=32
    ("INT8", "bf16", 200, 384, 8),
    ("INT8", "f32", 130, 256, 6),
    ("INT8_G64", "bf16", 96, 192, 8),
    ("MXINT8", "bf16", 257, 224, 8),
    ("MXINT8", "f32", 64, 160, 8),
    ("MXINT8", "bf16", 3000, 128, 6),       # rows past the resident ones stream from L2
]


@pytest.mark.parametrize("fmt_name,dtype,m,n,iters", CASES)
def test_solve_matches_oracle(dq, fmt_name, dtype, m, n, iters):
    W = _matrix(1000 + m + n, m, n, dtype)
    h, ora, _ = _check(dq, W, fmt_name, iters, f"{fmt_name}/{dtype}/{m}x{n}")
    if oracle_format(fmt_name).kind == "NVFP4":
        assert np.float32(h["tensor_scale"][0]) == ora["s_t"]
    assert_monotone(h["mse"], label=fmt_name)
    assert h["mse"][-1] <= h["mse"][0]


@pytest.mark.parametrize("fmt_name,m,n", [("NVFP4", 3000, 256), ("MXINT4", 8000, 64),
                                           ("INT4_G64", 2600, 128)])
def test_l2_streamed_rows_both_load_widths(dq, fmt_name, m, n):
    """Tall tiles keep only their top rows in shared memory and re-read the rest every pass:
    256-bit loads when every row starts 32-byte aligned, 128-bit loads otherwise (a row
    pitch of n + 8 bf16 elements). Both give identical results, and they match the oracle."""
    W = _matrix(4242 + m, m, n, "bf16")
    h = _run(dq, W, fmt_name, 8)
    padded = torch.zeros((m, n + 8), dtype=torch.bfloat16)
    padded[:, :n] = W
    view = padded.cuda()[:, :n]
    assert (view.stride(0) * 2) % 32 == 16
    out = dq.solve(view, fmt_name, 8)
    torch.cuda.synchronize()
    assert dq.last_device_error() == 0
    hp = to_host(out)
    for key in ("q_packed", "r", "c", "block_scales", "mse"):
        np.testing.assert_array_equal(hp[key], h[key], err_msg=key)
    _check(dq, W, fmt_name, 8, f"{fmt_name}/{m}x{n}/streamed")


def test_config1_tile_full(dq):
    cfg = wl.CONFIGS[1]
    W = wl.weight_host(cfg, 0, 0)
    h, ora, rep = _check(dq, W, "INT4", cfg.iters, "config1")
    assert h["mse"][0] / h["mse"][-1] > 4.0, rep


@pytest.mark.parametrize("fmt_name", ["INT4", "MXINT4", "MXFP4", "NVFP4", "INT8", "MXINT8"])
def test_iteration0_is_exact(dq, fmt_name):
    """iters = 0: single-scale RTN; every decision is on identical binary32 values."""
    W = _matrix(7, 300, 256, "bf16")
    h = _run(dq, W, fmt_name, 0)
    ora = S.solve(W.float().numpy().astype(np.float64), oracle_format(fmt_name), 0)
    compare_solve(h, ora, oracle_format(fmt_name), exact=True, label=fmt_name)
    np.testing.assert_array_equal(h["c"], np.ones(256, np.float32))
    np.testing.assert_array_equal(h["r"], ora["r"])


@pytest.mark.parametrize("fmt_name", ["INT4_G64", "MXINT4", "MXFP4", "NVFP4", "INT8_G64",
                                      "MXINT8"])
def test_warm_start_q_step_is_bit_exact(dq, fmt_name):
    """From the same binary32 state (r, c), the Q-step codes are identical and one further
    iteration agrees up to binary32-vs-binary64 summation."""
    fmt = oracle_format(fmt_name)
    W = _matrix(11, 256, 512, "bf16")
    Wd = W.float().numpy().astype(np.float64)
    ora5 = S.solve(Wd, fmt, 5)
    amax = None
    h0 = _run(dq, W, fmt_name, 0, r0=ora5["r"], c0=ora5["c"])
    o0 = S.solve(Wd, fmt, 0, r0=ora5["r"], c0=ora5["c"], amax=amax)
    compare_solve(h0, o0, fmt, exact=True, label="warm0")
    np.testing.assert_array_equal(h0["c"], ora5["c"])
    h1, o1, rep = _check(dq, W, fmt_name, 1, "warm1", r0=ora5["r"], c0=ora5["c"])
    assert rep["code_match"] == 1.0                        # the Q-step itself is exact
    assert rep["c_rel"] < 1e-6


def test_deterministic_and_batch_independent(dq):
    Ws = [_matrix(20 + i, 384, 512, "bf16") for i in range(3)]
    a = [to_host(o) for o in dq.solve_batched([w.cuda() for w in Ws], "NVFP4", 8)]
    b = [to_host(o) for o in dq.solve_batched([w.cuda() for w in Ws], "NVFP4", 8)]
    single = to_host(dq.solve(Ws[1].cuda(), "NVFP4", 8))
    for x, y in zip(a, b):
        for k in x:
            np.testing.assert_array_equal(x[k], y[k])
    for k in single:
        np.testing.assert_array_equal(single[k], a[1][k])


def test_batched_mixed_shapes(dq):
    shapes = [(256, 512), (128, 512), (256, 512), (64, 1024)]
    Ws = [_matrix(40 + i, m, n, "bf16") for i, (m, n) in enumerate(shapes)]
    outs = dq.solve_batched([w.cuda() for w in Ws], "MXFP4", 6)
    prev = dq.solve_batched([w.cuda() for w in Ws], "MXFP4", 5)
    fmt = oracle_format("MXFP4")
    for W, o, op in zip(Ws, outs, prev):
        Wd = torch_to_f64(W)
        compare_solve(to_host(o), oracle_solve(Wd, fmt, 6), fmt, W=Wd, h_prev=to_host(op),
                      label=str(W.shape))


def test_zero_matrix_rows_and_columns(dq):
    W = _matrix(50, 96, 128, "bf16")
    W[5, :] = 0
    W[:, 17] = 0
    W[40:48, 32:64] = 0
    for fmt_name in ["NVFP4", "MXINT4"]:
        h, _, _ = _check(dq, W, fmt_name, 6, "zeros")
        assert h["c"][17] == 1.0              # an all-zero column keeps its scale
    Z = torch.zeros(64, 64, dtype=torch.bfloat16)
    h = _run(dq, Z, "NVFP4", 3)
    assert np.all(h["mse"] == 0.0) and np.all(h["q_packed"] == 0)
    assert h["tensor_scale"][0] == 1.0


def test_nonfinite_input_is_reported(dq):
    W = _matrix(60, 64, 64, "bf16")
    W[3, 7] = float("nan")
    dq.solve(W.cuda(), "NVFP4", 2)
    assert dq.last_device_error() == 5            # DQ_ERR_NONFINITE
    assert dq.last_device_error() == 0            # cleared


def test_bad_warm_start_is_reported(dq):
    W = _matrix(61, 64, 64, "bf16")
    c0 = torch.full((64,), -1.0).cuda()
    dq.solve(W.cuda(), "MXFP4", 2, c0=c0)
    assert dq.last_device_error() == 1            # DQ_ERR_INVALID_ARG


def test_shape_errors_raise(dq):
    W = _matrix(62, 64, 100, "bf16").cuda()
    with pytest.raises(dq.DQError):
        dq.solve(W, "NVFP4", 2)
