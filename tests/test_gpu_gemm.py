"""The W4A4 GEMM on the tensor cores against the oracle's plain definition (B200).

Operands are the 4-bit codes and E4M3 block-scale codes the solver and the activation
quantizer produce. The tensor core accumulates in binary32, 64 elements per instruction, so
the bar is |y - y_oracle| <= (K/64 + 4) * 2^-23 * sum_j |x_hat w_hat| (one binary32
rounding per instruction and a few for the final scaling), elementwise.
"""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import gemm as G
from oracle import solver as S

pytestmark = pytest.mark.gpu
NV = F.make_format("NVFP4")


@pytest.fixture(scope="module")
def dq():
    import calibration_free_dual_b200 as pkg
    return pkg


def _operand(rng, rows, K, zero_frac=0.0):
    codes = rng.integers(0, 16, (rows, K)).astype(np.uint8)
    sc = rng.integers(1, 127, (rows, K // 16)).astype(np.uint8)
    if zero_frac:
        z = rng.random((rows, K // 16)) < zero_frac
        sc[z] = 0
        codes[np.repeat(z, 16, axis=1)] = 0
    return codes, sc


def _gpu(dq, xc, xs, sx, wc, ws, sw):
    dev = torch.device("cuda")
    x = dict(x_packed=torch.from_numpy(F.pack_codes(xc)).to(dev),
             scales=torch.from_numpy(xs).to(dev),
             tensor_scale=torch.tensor([sx], dtype=torch.float32, device=dev))
    w = dict(q_packed=torch.from_numpy(F.pack_codes(wc)).to(dev),
             block_scales=torch.from_numpy(ws).to(dev),
             tensor_scale=torch.tensor([sw], dtype=torch.float32, device=dev))
    y = dq.w4a4_gemm(x, w)
    torch.cuda.synchronize()
    assert dq.last_device_error() == 0
    return y.cpu().numpy().astype(np.float64)


def _check(y, xc, xs, sx, wc, ws, sw, K):
    ref = G.w4a4_gemm(xc, xs, sx, wc, ws, sw, NV)
    bound = (K / 64 + 4) * 2.0 ** -23 * G.abs_products(xc, xs, sx, wc, ws, sw, NV) + 1e-30
    err = np.abs(y - ref)
    assert np.all(err <= bound), (float((err / bound).max()), np.argwhere(err > bound)[:5])


@pytest.mark.parametrize("T,N,K", [(128, 128, 256), (256, 384, 1024), (200, 136, 320),
                                   (1, 8, 64), (130, 260, 4096),
                                   # 40 groups of 64 (a ragged 32-group re-layout chunk), an
                                   # output row pitch that is not a multiple of 4 floats
                                   (67, 130, 2560)])
def test_gemm_matches_oracle(dq, T, N, K):
    rng = np.random.default_rng(T * 7 + N + K)
    xc, xs = _operand(rng, T, K, zero_frac=0.05)
    wc, ws = _operand(rng, N, K)
    sx, sw = np.float32(0.03125), np.float32(0.0017)
    y = _gpu(dq, xc, xs, sx, wc, ws, sw)
    _check(y, xc, xs, sx, wc, ws, sw, K)


def test_gemm_on_the_solver_and_activation_outputs(dq):
    """Solve a weight in NVFP4, quantize an activation with its column scales, multiply:
    matches the oracle GEMM of the same codes, and approximates W x."""
    rng = np.random.default_rng(9)
    m, K, T = 384, 1024, 130
    w = rng.standard_t(4, (m, K)) * 0.014
    w[:, rng.choice(K, 4, replace=False)] *= 10.0
    W = torch.from_numpy(w.astype(np.float32)).to(torch.bfloat16).cuda()
    sol = dq.solve(W, "NVFP4", 8)
    X = rng.standard_normal((T, K)).astype(np.float32)
    X[:, rng.choice(K, 6, replace=False)] *= 50.0
    X[3] = 0.0
    Xt = torch.from_numpy(X).to(torch.bfloat16).cuda()
    act = dq.act_quant(Xt, "NVFP4", sol["c"])
    y = dq.w4a4_gemm(act, sol)
    torch.cuda.synchronize()
    assert dq.last_device_error() == 0
    y = y.cpu().numpy().astype(np.float64)
    xc = F.unpack_codes(act["x_packed"].cpu().numpy())
    xs = act["scales"].cpu().numpy()
    sx = act["tensor_scale"].cpu().numpy()[0]
    wc = F.unpack_codes(sol["q_packed"].cpu().numpy())
    ws = sol["block_scales"].cpu().numpy()
    sw = sol["tensor_scale"].cpu().numpy()[0]
    _check(y, xc, xs, sx, wc, ws, sw, K)
    assert np.all(y[3] == 0.0)
    ref = Xt.float().cpu().numpy().astype(np.float64) @ W.float().cpu().numpy().astype(np.float64).T
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel < 0.2, rel                      # 4-bit weights and activations


def test_gemm_rejects_bad_shapes(dq):
    f = dq.fmt_of("NVFP4")
    nul = None
    assert dq.dq_w4a4_gemm(nul, nul, nul, 8, nul, nul, nul, 8, 96, f, nul, 8, nul, 0, nul) == 2
    assert dq.dq_w4a4_gemm(nul, nul, nul, 8, nul, nul, nul, 8, 128, dq.fmt_of("MXFP4"), nul, 8,
                           nul, 0, nul) == 8
    assert dq.dq_w4a4_gemm_workspace_bytes(8, 8, 96) == 0


def _weight(dq, rng, N, K):
    """A solved NVFP4 weight (codes, block scales, tensor scale as dq_solve returns them)."""
    w = rng.standard_t(4, (N, K)) * 0.014
    W = torch.from_numpy(w.astype(np.float32)).to(torch.bfloat16).cuda()
    return dq.solve(W, "NVFP4", 4)


@pytest.mark.parametrize("T,N,K,ldx_pad,with_c", [(130, 260, 4096, 0, True), (1, 8, 64, 0, True),
                                                  (256, 384, 1024, 64, True),
                                                  (67, 130, 2560, 0, False),
                                                  (200, 136, 320, 32, True)])
def test_linear_is_act_quant_then_gemm_bit_for_bit(dq, T, N, K, ldx_pad, with_c):
    """dq_w4a4_linear (one quantization pass writing the tensor core's layouts, then the GEMM)
    equals dq_act_quant followed by dq_w4a4_gemm exactly: ragged token blocks (their padded
    scale rows zero), a strided X, no c, an output pitch that is not a multiple of 4 floats."""
    rng = np.random.default_rng(T + 3 * N + K)
    sol = _weight(dq, rng, N, K)
    X = rng.standard_normal((T, K + ldx_pad)).astype(np.float32)
    X[:, rng.choice(K, min(6, K), replace=False)] *= 50.0
    Xd = torch.from_numpy(X).to(torch.bfloat16).cuda()[:, :K]
    c = sol["c"] if with_c else None
    y1 = dq.w4a4_linear(Xd, sol, c)
    act = dq.act_quant(Xd, "NVFP4", c)
    y2 = dq.w4a4_gemm(act, sol)
    torch.cuda.synchronize()
    assert dq.last_device_error() == 0
    assert torch.equal(y1, y2)


def test_linear_matches_the_oracle_composition(dq):
    """Against the oracle: its activation quantizer on fl32(X * c), then its GEMM of the two
    sets of codes, within the GEMM's binary32 accumulation bound."""
    rng = np.random.default_rng(21)
    T, N, K = 150, 256, 1024
    sol = _weight(dq, rng, N, K)
    X = rng.standard_normal((T, K)).astype(np.float32)
    X[:, rng.choice(K, 6, replace=False)] *= 50.0
    Xt = torch.from_numpy(X).to(torch.bfloat16)
    y = dq.w4a4_linear(Xt.cuda(), sol, sol["c"])
    torch.cuda.synchronize()
    assert dq.last_device_error() == 0
    y = y.cpu().numpy().astype(np.float64)
    from oracle import actquant as AQ
    a = AQ.act_quant(Xt.float().numpy(), NV, sol["c"].cpu().numpy())
    wc = F.unpack_codes(sol["q_packed"].cpu().numpy())
    ws = sol["block_scales"].cpu().numpy()
    sw = sol["tensor_scale"].cpu().numpy()[0]
    _check(y, a["codes"], a["scale_codes"], a["s_t"], wc, ws, sw, K)
