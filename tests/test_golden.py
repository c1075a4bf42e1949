"""Hand-worked examples of the dual-scale BCD solve (tests/golden/worked_examples.txt).

The pages print no worked example, so these were derived by hand from the method's
definition (DualQuant abstract: closed-form block updates of W ~ diag(r) Q diag(c); the
acceptodds.com abstract: black-box quantizer, scales projected after every update; Figure 1
(b): iteration 0 is single-scale round-to-nearest; Figure 2 (b): the normalised-MSE trace).
Each example exercises the format's element ties, its scale projection, both closed forms
and the trace with exact dyadic numbers (INT4, MXFP4, NVFP4, MXINT4 and the 8-bit INT8).
The oracle is checked against all of them on the CPU with 4-column blocks; the CUDA path
against the INT4, MXFP4 and NVFP4 ones with every row padded by zero columns to the format's
real block length (zeros change no block maximum or sum).
"""
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import formats as F
from oracle import solver as S

HERE = os.path.dirname(os.path.abspath(__file__))
FIXTURE = os.path.join(HERE, "golden", "worked_examples.txt")
REAL_BLOCK = {"INT4": 64, "MXFP4": 32, "NVFP4": 16}


def _num(tok: str) -> Fraction:
    if tok.lower().startswith("0x"):
        return Fraction(int(tok, 16))
    if "e" in tok.lower() or ("." in tok):
        return Fraction(float(tok))
    return Fraction(tok)


def _load():
    ex, cur = {}, None
    with open(FIXTURE) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("["):
                cur = ex.setdefault(line.strip("[]"), {})
                continue
            key, val = line.split(":", 1)
            key, val = key.strip(), val.strip()
            if key == "fmt":
                cur[key] = val
            elif key.endswith("_codes") or key.endswith("_bits"):
                cur[key] = [int(t, 0) for t in val.split()]
            elif "|" in val:
                cur[key] = [[_num(t) for t in row.split()] for row in val.split("|")]
            else:
                vals = [_num(t) for t in val.split()]
                cur[key] = vals[0] if len(vals) == 1 and key.startswith(("mse", "s_t", "qchange")) else vals
    return ex


EXAMPLES = _load()


def _arr(rows):
    return np.array([[float(v) for v in row] for row in rows], dtype=np.float64)


def _bits32(x):
    return [int(v) for v in np.asarray(x, dtype=np.float32).view(np.uint32)]


def test_fixture_is_consistent():
    """The fixture's own arithmetic: W has 2 rows of 4; every example is complete."""
    assert set(EXAMPLES) == {"INT4", "MXFP4", "NVFP4", "MXINT4", "INT8", "QCHANGE"}
    for ex in EXAMPLES.values():
        assert len(ex["W"]) == 2 and all(len(r) == 4 for r in ex["W"])
        for k in ("r0_codes", "q0", "mse0", "r1_codes", "N1", "D1", "c1_bits", "mse1"):
            assert k in ex


@pytest.mark.parametrize("name", sorted(EXAMPLES))
def test_oracle_iteration0_is_the_hand_rtn(name):
    ex = EXAMPLES[name]
    fmt = F.make_format(ex["fmt"], 4)
    out = S.solve(_arr(ex["W"]), fmt, 0)
    assert [int(v) for v in out["r_codes"][:, 0]] == ex["r0_codes"]
    np.testing.assert_array_equal(out["q"], _arr(ex["q0"]))
    assert out["mse"][0] == pytest.approx(float(ex["mse0"]), rel=1e-15)
    if "s_t" in ex:
        assert out["s_t"] == np.float32(float(ex["s_t"]))


@pytest.mark.parametrize("name", sorted(EXAMPLES))
def test_oracle_iteration1_is_the_hand_update(name):
    ex = EXAMPLES[name]
    fmt = F.make_format(ex["fmt"], 4)
    W = _arr(ex["W"])
    out = S.solve(W, fmt, 1)
    assert [int(v) for v in out["r_codes"][:, 0]] == ex["r1_codes"]
    # the hand sums of the c-step, formed from the hand state (r1, q0)
    N, D = S.c_step_sums(W, _arr(ex["q0"]), out["r"], 4)
    assert [Fraction(v) for v in N] == ex["N1"]
    assert [Fraction(v) for v in D] == ex["D1"]
    assert _bits32(out["c"]) == ex["c1_bits"]
    np.testing.assert_array_equal(out["q"], _arr(ex["q0"]))
    assert out["mse"][1] == pytest.approx(float(ex["mse1"]), rel=1e-12, abs=1e-300)
    assert out["mse"][1] <= out["mse"][0]


def test_oracle_exact_fit_is_a_fixed_point():
    ex = EXAMPLES["MXFP4"]
    out = S.solve(_arr(ex["W"]), F.make_format("MXFP4", 4), 2)
    np.testing.assert_array_equal(out["q"], _arr(ex["q2"]))
    assert out["mse"][1] == 0.0 and out["mse"][2] == 0.0


def _qchange_variants(q_prev, q_now, fmt):
    """qchange[t]^2 by the definition and by three plausible mistakes: normalising by the new
    iterate, using element codes instead of values, and forgetting the square root."""
    d = float(np.sum((q_now - q_prev) ** 2))
    right = d / float(np.sum(q_prev ** 2))
    cp = F.round_elem(q_prev.astype(np.float32), fmt)[0].astype(np.float64)
    cn = F.round_elem(q_now.astype(np.float32), fmt)[0].astype(np.float64)
    return right, {"new-iterate norm": d / float(np.sum(q_now ** 2)),
                   "codes": float(np.sum((cn - cp) ** 2)) / float(np.sum(cp ** 2)),
                   "unrooted": right ** 2}


def test_oracle_qchange_is_the_hand_value():
    """Figure 2 (a)'s relative change of Q-hat on the hand example whose W[1, 0] code moves
    between iterations 1 and 2: qchange = [0, 0, sqrt(1/429)] exactly, with the hand state of
    the second iteration (codes, r-step, c-step sums, c bits, MSE)."""
    ex = EXAMPLES["QCHANGE"]
    fmt = F.make_format(ex["fmt"], 4)
    W = _arr(ex["W"])
    out = S.solve(W, fmt, 2)
    np.testing.assert_array_equal(out["q"], _arr(ex["q2"]))
    assert [int(v) for v in out["r_codes"][:, 0]] == ex["r2_codes"]
    N, D = S.c_step_sums(W, _arr(ex["q2"]), out["r"], 4)
    assert [Fraction(v) for v in N] == ex["N2"]
    assert [Fraction(v) for v in D] == ex["D2"]
    assert _bits32(out["c"]) == ex["c2_bits"]
    assert out["mse"][2] == pytest.approx(float(ex["mse2"]), rel=1e-12)
    qc = out["qchange"]
    assert qc[0] == 0.0 and qc[1] == 0.0
    assert qc[2] ** 2 == pytest.approx(float(ex["qchange2_sq"]), rel=1e-14)
    assert qc[2] == pytest.approx(float(ex["qchange2_sq"]) ** 0.5, rel=1e-15)


def test_qchange_pin_separates_the_plausible_mistakes():
    """The pinned value tells the definition apart from each mistake the oracle could make."""
    ex = EXAMPLES["QCHANGE"]
    fmt = F.make_format(ex["fmt"], 4)
    right, wrong = _qchange_variants(_arr(ex["q0"]), _arr(ex["q2"]), fmt)
    assert right == pytest.approx(float(ex["qchange2_sq"]), rel=1e-15)
    for name, v in wrong.items():
        assert abs(v - right) > 0.01 * right, name


def _padded(ex):
    B = REAL_BLOCK[ex["fmt"]]
    W = np.zeros((2, B), dtype=np.float64)
    W[:, :4] = _arr(ex["W"])
    return W


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["INT4", "MXFP4", "NVFP4"])
def test_cuda_path_reproduces_the_hand_example(name):
    import torch
    import calibration_free_dual_b200 as dq

    ex = EXAMPLES[name]
    fmt_name = "INT4_G64" if ex["fmt"] == "INT4" else ex["fmt"]
    W = torch.from_numpy(_padded(ex).astype(np.float32)).cuda()
    fmt = F.make_format(ex["fmt"], REAL_BLOCK[ex["fmt"]])
    for iters in (0, 1):
        out = dq.solve(W, fmt_name, iters)
        torch.cuda.synchronize()
        assert dq.last_device_error() == 0
        scodes = out["block_scales"].cpu().numpy().astype(np.int64)[:, 0]
        if ex["fmt"] == "INT4":
            scodes = scodes & 0xFFFF
        assert [int(v) for v in scodes] == ex["r0_codes" if iters == 0 else "r1_codes"]
        codes = F.unpack_codes(out["q_packed"].cpu().numpy())
        q = F.decode_elem(codes, fmt)
        np.testing.assert_array_equal(q[:, :4], _arr(ex["q0"]))
        assert not q[:, 4:].any()
        mse = out["mse"].cpu().numpy()
        assert mse[0] == pytest.approx(float(ex["mse0"]), rel=1e-6)
        if iters == 1:
            c = out["c"].cpu().numpy()
            assert _bits32(c[:4]) == ex["c1_bits"]
            assert np.all(c[4:] == 1.0)
            assert abs(mse[1] - float(ex["mse1"])) <= max(1e-4 * float(ex["mse1"]), 1e-6)
        if "s_t" in ex:
            assert out["tensor_scale"].cpu().numpy()[0] == np.float32(float(ex["s_t"]))


@pytest.mark.gpu
def test_cuda_qchange_trace_is_the_hand_value():
    """The CUDA path's Q-change trace (dq_solve_batched_ex) on the hand example padded to the
    real MXFP4 block: [0, 0, sqrt(1/429)] (both of its sums are exact), the codes of the
    second iteration, and the other outputs unchanged by asking for the trace."""
    import torch
    import calibration_free_dual_b200 as dq

    ex = EXAMPLES["QCHANGE"]
    W = torch.from_numpy(_padded(ex).astype(np.float32)).cuda()
    fmt = F.make_format(ex["fmt"], REAL_BLOCK[ex["fmt"]])
    out = dq.solve_batched([W], ex["fmt"], 2, qchange=True)[0]
    torch.cuda.synchronize()
    assert dq.last_device_error() == 0
    qc = out["qchange"].cpu().numpy()
    assert qc[0] == 0.0 and qc[1] == 0.0
    assert qc[2] == pytest.approx(float(ex["qchange2_sq"]) ** 0.5, rel=1e-15)
    q = F.decode_elem(F.unpack_codes(out["q_packed"].cpu().numpy()), fmt)
    np.testing.assert_array_equal(q[:, :4], _arr(ex["q2"]))
    assert _bits32(out["c"].cpu().numpy()[:4]) == ex["c2_bits"]
