"""Two shortcuts the kernels take with bf16 block scales, checked against their bounds (host).

The solve kernel's r-step for the bf16-scale formats (INT4, INT8) forms the least-squares
quotient num/den of a block in binary32 first: each lane accumulates its 16 elements as two
chains of 8 fused multiply-adds (even and odd elements) on products q*c rounded to binary32,
adds the two chains, and the lanes of the block combine by an xor butterfly. Every term is
non-negative, since a code has the sign of its weight, so num and den carry at most 13 and 14
binary32 roundings of relative error and the correctly rounded quotient at most 28: under 28
ulps. The kernel trusts the binary32 quotient when it lies more than 128 ulps from a bf16
rounding point and takes the sums again in binary64 otherwise.

This emulates that summation order in NumPy (binary32 with the fused multiply-add formed in
binary64, where the product is exact) on blocks of the shapes and distributions the solver
meets, and checks the bound and that the bf16 decision outside the band equals the decision
on the exact quotient (80-bit sums, where every product w*q*c is exact).
"""
import numpy as np
import pytest

F32, F64, LD = np.float32, np.float64, np.longdouble


def _fma32(a, b, acc):
    return (a.astype(F64) * b.astype(F64) + acc.astype(F64)).astype(F32)


def _kernel_sums(w, q, c):
    """num, den of each block (rows of [nblk, B]) in the kernel's binary32 order."""
    nblk, B = w.shape
    lanes = B // 16
    qc = (q.astype(F32) * c.astype(F32)).astype(F32)
    num = np.zeros((nblk, lanes), F32)
    den = np.zeros((nblk, lanes), F32)
    for lane in range(lanes):
        nx = np.zeros(nblk, F32); ny = np.zeros(nblk, F32)
        dx = np.zeros(nblk, F32); dy = np.zeros(nblk, F32)
        for p in range(8):
            j = lane * 16 + 2 * p
            nx = _fma32(w[:, j], qc[:, j], nx)
            ny = _fma32(w[:, j + 1], qc[:, j + 1], ny)
            dx = _fma32(qc[:, j], qc[:, j], dx)
            dy = _fma32(qc[:, j + 1], qc[:, j + 1], dy)
        num[:, lane] = nx + ny
        den[:, lane] = dx + dy
    off = 1
    while off < lanes:
        num = num + num[:, np.arange(lanes) ^ off]
        den = den + den[:, np.arange(lanes) ^ off]
        off <<= 1
    assert np.all(num == num[:, :1]) and np.all(den == den[:, :1])   # every lane agrees
    return num[:, 0], den[:, 0]


def _blocks(rng, nblk, B, qmax, kind):
    if kind == "normal":
        w = rng.standard_normal((nblk, B))
    elif kind == "t4":
        w = rng.standard_t(4, (nblk, B))
    else:                                   # mixed magnitudes inside a block
        w = rng.standard_normal((nblk, B)) * np.exp2(rng.integers(-20, 4, (nblk, B)))
    w = (w * 0.02).astype(F32)
    c = np.exp(rng.normal(0.0, 0.7, (nblk, B))).astype(F32)
    x = w.astype(F64) / c.astype(F64)
    r = np.abs(x).max(axis=1, keepdims=True) / qmax * rng.uniform(0.6, 1.2, (nblk, 1))
    q = np.clip(np.rint(x / r), -qmax, qmax).astype(F32)
    return w, q, c


def _bf16_rn(v32):
    u = v32.view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint32)


@pytest.mark.parametrize("B,qmax", [(128, 7), (64, 7), (128, 127), (64, 127)])
@pytest.mark.parametrize("kind", ["normal", "t4", "mixed"])
def test_binary32_block_sums_within_bound(B, qmax, kind):
    rng = np.random.default_rng(B * 1000 + qmax + len(kind))
    w, q, c = _blocks(rng, 4000, B, qmax, kind)
    num32, den32 = _kernel_sums(w, q, c)
    ok = den32 > 0
    v32 = (num32[ok].astype(F64) / den32[ok].astype(F64)).astype(F32)   # one rounding of the ratio
    # the exact quotient: every w*q*c is exact in the 64-bit significand, the sums nearly so
    wq = w[ok].astype(LD) * q[ok].astype(LD)
    cl = c[ok].astype(LD)
    num = (wq * cl).sum(axis=1)
    den = ((q[ok].astype(LD) * cl) ** 2).sum(axis=1)
    assert np.all(wq >= 0)                  # every term non-negative
    v = num / den
    ulps = np.abs(v32.astype(LD) - v) / np.spacing(v32).astype(LD)
    assert ulps.max() < 28, float(ulps.max())
    # outside the band the bf16 decision is the exact quotient's
    lo = v32.view(np.uint32) & 0xFFFF
    sure = np.abs(lo.astype(np.int64) - 0x8000) > 128
    exact32 = v.astype(F64).astype(F32)
    assert np.array_equal(_bf16_rn(v32)[sure], _bf16_rn(exact32)[sure])
    assert sure.mean() > 0.99


@pytest.mark.parametrize("Q", [7, 127])
def test_bf16_scale_codes_stay_in_range_without_a_clamp(Q):
    """The activation quantizer rounds x * fl32(1/s) to an integer code without clamping it when
    s is a bf16 block scale bf16(fl32(a/Q)), a the block's largest |x|: the quotient stays below
    Q + 1/2. Checked for every binary32 a in [1, 2) (the ratio repeats in every binade above
    the bf16 scale's lower clamp, which only makes s larger)."""
    a = np.arange(0x3F800000, 0x40000000, dtype=np.uint64).astype(np.uint32).view(F32)
    v = (a.astype(F64) / Q).astype(F32)
    u = v.view(np.uint32).astype(np.uint64)
    s = (((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16).astype(np.uint32).view(F32)
    inv = (1.0 / s.astype(F64)).astype(F32)
    y = (a.astype(F64) * inv.astype(F64)).astype(F32)
    assert float(y.max()) < Q + 0.5
