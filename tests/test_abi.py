"""The C ABI library loads and exports what include/dq.h declares; host-side validation
rejects bad arguments before any CUDA call (CPU only, no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def dq():
    from calibration_free_dual_b200 import build
    build.build()
    import calibration_free_dual_b200 as pkg
    return pkg


def _declared():
    src = open(os.path.join(ROOT, "include", "dq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"DQ_API\s+[\w\s\*]+?\b(dq_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ["dq_solve", "dq_solve_batched", "dq_solve_workspace_bytes", "dq_act_quant",
                 "dq_act_quant_workspace_bytes", "dq_encode", "dq_decode",
                 "dq_last_device_error", "dq_status_string", "dq_solve_max_rows"]:
        assert must in names


def test_library_exports_every_declared_symbol(dq):
    lib = ctypes.CDLL(dq._lib.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    # and nothing else with the dq_ prefix is missing from the binding
    for name in _declared():
        assert name in dq._lib.SIGNATURES, name


def test_exports_are_only_the_c_abi(dq):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", dq._lib.LIB_PATH],
                         stdout=subprocess.PIPE, text=True).stdout
    text_syms = [l.split()[-1] for l in out.splitlines() if " T " in l]
    assert sorted(text_syms) == _declared()


def test_status_strings(dq):
    assert dq.dq_status_string(0) == b"DQ_OK"
    assert dq.dq_status_string(2) == b"DQ_ERR_SHAPE"
    assert dq.dq_status_string(99) == b"DQ_ERR_UNKNOWN"


def test_validation_happens_before_cuda(dq):
    f = dq.fmt_of("NVFP4")
    nul = None
    # n not a multiple of the block length
    assert dq.dq_solve(nul, 1, 64, 100, 100, f, 4, nul, nul, nul, nul, nul, nul, nul, nul,
                       nul, 0, nul) == 2
    # null W with a valid shape
    assert dq.dq_solve(nul, 1, 64, 128, 128, f, 4, nul, nul, nul, nul, nul, nul, nul, nul,
                       nul, 0, nul) == 1
    # bad format / dtype
    bad = dq.dq_format(3, 32)
    assert dq.dq_solve(nul, 1, 64, 128, 128, bad, 4, nul, nul, nul, nul, nul, nul, nul, nul,
                       nul, 0, nul) == 3
    assert dq.dq_solve(nul, 7, 64, 128, 128, f, 4, nul, nul, nul, nul, nul, nul, nul, nul,
                       nul, 0, nul) == 3
    # negative iterations, ldw < n
    assert dq.dq_solve(nul, 1, 64, 128, 128, f, -1, nul, nul, nul, nul, nul, nul, nul, nul,
                       nul, 0, nul) == 1
    assert dq.dq_solve(nul, 1, 64, 128, 64, f, 4, nul, nul, nul, nul, nul, nul, nul, nul,
                       nul, 0, nul) == 1
    # act quant shape / workspace checks
    assert dq.dq_act_quant(nul, 1, 8, 100, 100, nul, f, nul, nul, nul, nul, 0, nul) == 2
    assert dq.dq_act_quant(nul, 1, 8, 128, 128, nul, f, nul, nul, nul, nul, 0, nul) == 1
    assert dq.dq_encode(nul, 4, 9, nul, nul) == 3
    assert dq.dq_decode(nul, -1, 1, nul, nul) == 1


def test_workspace_bytes_and_limits(dq):
    f = dq.fmt_of("NVFP4")
    m = (ctypes.c_int64 * 2)(4096, 14336)
    n = (ctypes.c_int64 * 2)(4096, 4096)
    one = dq.dq_solve_workspace_bytes(1, m, n, f, 16)
    two = dq.dq_solve_workspace_bytes(2, m, n, f, 16)
    assert 0 < one < two
    assert dq.dq_solve_workspace_bytes(1, m, (ctypes.c_int64 * 1)(100), f, 16) == 0
    assert dq.dq_solve_max_rows(4096, f, 1) >= 14336            # 8B-shaped gate/up fit
    assert dq.dq_solve_max_rows(4096, dq.fmt_of("MXFP4"), 1) >= 11008
    assert dq.dq_solve_max_rows(512, dq.fmt_of("INT4"), 0) >= 512
    assert dq.dq_act_quant_workspace_bytes(8192, 4096, f) > 0


def test_no_cpu_fallback(dq):
    import torch
    with pytest.raises(TypeError):
        dq.solve(torch.zeros(16, 32), "NVFP4", 2)
    with pytest.raises(TypeError):
        dq.act_quant(torch.zeros(4, 32), "NVFP4")


def test_solve_options_validation_and_workspace(dq):
    """dq_solve_batched_ex: an unknown update mode or a null Q-change pointer is rejected
    before anything reaches CUDA; the Q-change trace needs more workspace."""
    f = dq.fmt_of("MXFP4")
    m = (ctypes.c_int64 * 1)(512)
    n = (ctypes.c_int64 * 1)(2048)
    plain = dq.dq_solve_workspace_bytes(1, m, n, f, 16)
    both = dq._lib.dq_solve_options(dq.DQ_UPDATE_BOTH, None)
    assert dq.dq_solve_workspace_bytes_ex(1, m, n, f, 16, ctypes.byref(both)) == plain
    assert dq.dq_solve_workspace_bytes_ex(1, m, n, f, 16, None) == plain
    qptr = (ctypes.c_void_p * 1)(0x1000)
    traced = dq._lib.dq_solve_options(dq.DQ_UPDATE_ROW_ONLY, qptr)
    assert dq.dq_solve_workspace_bytes_ex(1, m, n, f, 16, ctypes.byref(traced)) > plain
    mats = (dq.dq_matrix * 1)()
    mats[0] = dq.dq_matrix(0x1000, 512, 2048, 2048, None, None, 0x1000, 0x1000, 0x1000,
                           0x1000, 0x1000, 0x1000)
    bad_mode = dq._lib.dq_solve_options(5, None)
    assert dq.dq_solve_batched_ex(mats, 1, dq.DQ_BF16, f, 16, ctypes.byref(bad_mode), None, 0,
                                  None) == 1
    null_trace = dq._lib.dq_solve_options(dq.DQ_UPDATE_BOTH, (ctypes.c_void_p * 1)(None))
    assert dq.dq_solve_batched_ex(mats, 1, dq.DQ_BF16, f, 16, ctypes.byref(null_trace), None,
                                  0, None) == 1


def test_linear_validation_and_workspace(dq):
    """dq_w4a4_linear: format, shape, pointer and workspace checks before any CUDA call; the
    workspace holds the quantized activation and both operands' scale factors."""
    nv, mx = dq.fmt_of("NVFP4"), dq.fmt_of("MXFP4")
    nul = None
    assert dq.dq_w4a4_linear_workspace_bytes(130, 260, 96, nv) == 0          # K % 64
    assert dq.dq_w4a4_linear_workspace_bytes(130, 260, 4096, mx) == 0        # NVFP4 only
    need = dq.dq_w4a4_linear_workspace_bytes(130, 260, 4096, nv)
    # codes 130 x 2048, activation scale factors 2 blocks of 128 rows, weight's 3 blocks
    assert need >= 130 * 2048 + (256 + 384) * 256
    assert dq.dq_w4a4_linear(nul, 1, 8, 96, 96, nul, nul, nul, nul, 8, nv, nul, 8, nul, 0,
                             nul) == 2
    assert dq.dq_w4a4_linear(nul, 1, 8, 128, 128, nul, nul, nul, nul, 8, mx, nul, 8, nul, 0,
                             nul) == 8
    assert dq.dq_w4a4_linear(nul, 1, 8, 128, 128, nul, nul, nul, nul, 8, nv, nul, 8, nul, 0,
                             nul) == 1
    assert dq.dq_w4a4_linear(nul, 9, 8, 128, 128, nul, nul, nul, nul, 8, nv, nul, 8, nul, 0,
                             nul) == 3
    assert dq.dq_w4a4_linear(0x1000, 1, 8, 128, 64, nul, 0x1000, 0x1000, 0x1000, 8, nv,
                             0x1000, 8, nul, 0, nul) == 1                      # ldx < K
    assert dq.dq_w4a4_linear(0x1000, 1, 8, 128, 128, nul, 0x1000, 0x1000, 0x1000, 8, nv,
                             0x1000, 8, nul, 0, nul) == 4                      # no workspace


def test_act_quant_validation_before_cuda(dq):
    """Every malformed dq_act_quant call is refused on the host, before anything is queued
    (the pointers below are never dereferenced: each call fails one check)."""
    f = dq.fmt_of("NVFP4")
    P = ctypes.c_void_p
    X, c, xq, sc, ts, ws = P(0x10000), P(0x20000), P(0x30000), P(0x40000), P(0x50000), P(0x60000)
    nul = None
    # zero tokens: nothing to do, success without touching any pointer
    assert dq.dq_act_quant(nul, 1, 0, 128, 128, nul, f, nul, nul, nul, nul, 0, nul) == 0
    # ldx < n, negative tokens, unknown dtype
    assert dq.dq_act_quant(X, 1, 8, 128, 64, c, f, xq, sc, ts, ws, 256, nul) == 1
    assert dq.dq_act_quant(X, 1, -1, 128, 128, c, f, xq, sc, ts, ws, 256, nul) == 1
    assert dq.dq_act_quant(X, 9, 8, 128, 128, c, f, xq, sc, ts, ws, 256, nul) == 3
    # NVFP4 needs the tensor-scale output
    assert dq.dq_act_quant(X, 1, 8, 128, 128, c, f, xq, sc, nul, ws, 256, nul) == 1
    # X not 16-byte aligned, or a row pitch that is not a multiple of 16 bytes
    assert dq.dq_act_quant(P(0x10008), 1, 8, 128, 128, c, f, xq, sc, ts, ws, 256, nul) == 1
    assert dq.dq_act_quant(X, 1, 8, 128, 132, c, f, xq, sc, ts, ws, 256, nul) == 1
    # c not 16-byte aligned; codes not 4-byte aligned (8 for the 8-bit formats)
    assert dq.dq_act_quant(X, 1, 8, 128, 128, P(0x20004), f, xq, sc, ts, ws, 256, nul) == 1
    assert dq.dq_act_quant(X, 1, 8, 128, 128, c, f, P(0x30002), sc, ts, ws, 256, nul) == 1
    f8 = dq.fmt_of("MXINT8")
    assert dq.dq_act_quant(X, 1, 8, 128, 128, c, f8, P(0x30004), sc, ts, ws, 256, nul) == 1
    # missing or short workspace
    assert dq.dq_act_quant(X, 1, 8, 128, 128, c, f, xq, sc, ts, nul, 256, nul) == 4
    assert dq.dq_act_quant(X, 1, 8, 128, 128, c, f, xq, sc, ts, ws, 3, nul) == 4
