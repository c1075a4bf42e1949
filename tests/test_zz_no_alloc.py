"""dq_solve_noalloc: the solve for callers that cannot allocate device memory.

Hosts that own all device memory through their own pool allocator cannot let a library
call cudaMalloc; dq_solve_noalloc takes its scratch from a fixed array inside libdq.so
instead of a workspace argument. These tests call it through the C ABI and check that calls
in a row give exactly what dq_solve (caller-allocated workspace) gives. Kept in a file of its
own, collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests._parity import to_host


@pytest.fixture(scope="module")
def dq():
    import calibration_free_dual_b200 as pkg
    return pkg


def _matrix(seed, m, n):
    rng = np.random.default_rng(seed)
    w = rng.standard_t(4, (m, n)) * 0.014
    w[:, rng.choice(n, 3, replace=False)] *= 10.0
    return torch.from_numpy(w.astype(np.float32)).to(torch.bfloat16)


def _noalloc(dq, W, fmt_name, iters):
    """One dq_solve_noalloc call through the C ABI; outputs allocated by the test."""
    f = dq.fmt_of(fmt_name)
    m, n = W.shape
    o = dq.api.solve_outputs(m, n, f, iters, W.device)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = dq.dq_solve_noalloc(p(W), dq.DQ_BF16, m, n, W.stride(0), f, iters, None, None,
                             p(o["q_packed"]), p(o["r"]), p(o["c"]), p(o["block_scales"]),
                             p(o["tensor_scale"]), p(o["mse"]),
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, o


KEYS = ("q_packed", "r", "c", "block_scales", "tensor_scale", "mse")


@pytest.mark.gpu
@pytest.mark.parametrize("fmt_name", ["NVFP4", "MXFP4", "INT4"])
def test_noalloc_matches_dq_solve_on_two_calls(dq, fmt_name):
    """dq_solve_noalloc runs the same plan as dq_solve, so its outputs are bit-identical to a
    dq_solve call with a caller-allocated workspace; calls in a row (two shapes, a call in
    another format in between, then the first shape again) share the fixed scratch and must
    leave nothing behind that changes a later result."""
    Wa = _matrix(1, 384, 512).cuda()
    Wb = _matrix(2, 200, 256).cuda()
    other = "MXINT4" if fmt_name != "MXINT4" else "NVFP4"
    refs = {}
    for key, W, f in (("a", Wa, fmt_name), ("b", Wb, fmt_name), ("o", Wb, other)):
        refs[key] = to_host(dq.solve(W, f, 8))
    for key, W, f in (("a", Wa, fmt_name), ("b", Wb, fmt_name), ("o", Wb, other),
                      ("a", Wa, fmt_name)):
        st, out = _noalloc(dq, W, f, 8)
        assert st == 0, dq.dq_status_string(st)
        torch.cuda.synchronize()
        assert dq.last_device_error() == 0
        h = to_host(out)
        for k in KEYS:
            if k == "tensor_scale" and f != "NVFP4":
                continue                       # written by the NVFP4 solve only
            np.testing.assert_array_equal(h[k], refs[key][k], err_msg=f"{fmt_name}/{key}/{k}")


def test_noalloc_rejects_shapes_beyond_its_scratch(dq):
    f = dq.fmt_of("NVFP4")
    m, n, iters = 64, 16 * 4096, 200           # 4096 tiles x 202 fp64 partials > 4 MiB
    ms, ns = (ctypes.c_int64 * 1)(m), (ctypes.c_int64 * 1)(n)
    assert dq.dq_solve_workspace_bytes(1, ms, ns, f, iters) > dq._lib.DQ_NOALLOC_SCRATCH_BYTES
    nul = None
    st = dq.dq_solve_noalloc(nul, dq.DQ_BF16, m, n, n, f, iters, nul, nul, nul, nul, nul, nul,
                             nul, nul, nul)
    assert st == 4                                 # DQ_ERR_WORKSPACE, nothing launched
