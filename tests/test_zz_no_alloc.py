"""dq_solve_noalloc: the solve for callers that cannot allocate device memory.

Hosts that own all device memory through their own pool allocator cannot let a library
call cudaMalloc; dq_solve_noalloc takes its scratch from a fixed array inside libdq.so
instead of a workspace argument. These tests call it through the C ABI and check that two
calls in a row give what dq_solve (caller-allocated workspace) gives, within the parity
tolerances used by the other solver tests. Kept in a file of its own, collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import formats as F
from tests._parity import compare_solve, oracle_format, to_host


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


def _as_reference(h, fmt):
    """A dq_solve result in the form the parity comparison expects."""
    codes = F.unpack_codes(h["q_packed"])
    sc = h["block_scales"].view(np.uint16) if fmt.scale == "bf16" else h["block_scales"]
    return dict(codes=codes, q=F.decode_elem(codes, fmt), r_codes=sc.astype(np.int64),
                c=h["c"].astype(np.float32), mse=h["mse"])


@pytest.mark.gpu
@pytest.mark.parametrize("fmt_name", ["NVFP4", "MXFP4", "INT4"])
def test_noalloc_matches_dq_solve_on_two_calls(dq, fmt_name):
    fmt = oracle_format(fmt_name)
    Wa = _matrix(1, 384, 512).cuda()
    Wb = _matrix(2, 200, 256).cuda()
    refs = {}
    for key, W in (("a", Wa), ("b", Wb)):
        refs[key] = to_host(dq.solve(W, fmt_name, 8))
    # two calls in a row on the shared scratch (different shapes), then the first again
    for key, W in (("a", Wa), ("b", Wb), ("a", Wa)):
        st, out = _noalloc(dq, W, fmt_name, 8)
        assert st == 0, dq.dq_status_string(st)
        torch.cuda.synchronize()
        assert dq.last_device_error() == 0
        h = to_host(out)
        compare_solve(h, _as_reference(refs[key], fmt), fmt, label=f"noalloc/{fmt_name}/{key}")
        if fmt.kind == "NVFP4":
            assert h["tensor_scale"][0] == refs[key]["tensor_scale"][0]


def test_noalloc_rejects_shapes_beyond_its_scratch(dq):
    f = dq.fmt_of("NVFP4")
    m, n, iters = 64, 16 * 4096, 200           # 4096 tiles x 202 fp64 partials > 4 MiB
    ms, ns = (ctypes.c_int64 * 1)(m), (ctypes.c_int64 * 1)(n)
    assert dq.dq_solve_workspace_bytes(1, ms, ns, f, iters) > dq._lib.DQ_NOALLOC_SCRATCH_BYTES
    nul = None
    st = dq.dq_solve_noalloc(nul, dq.DQ_BF16, m, n, n, f, iters, nul, nul, nul, nul, nul, nul,
                             nul, nul, nul)
    assert st == 4                                 # DQ_ERR_WORKSPACE, nothing launched
