"""Pins for the oracle's format tables and roundings (CPU only).

Each codec is checked against something other than itself: torch's float8_e4m3fn /
float8_e8m0fnu / bfloat16 conversions (library routines), the bit-level definition of the
format, or a brute-force nearest-value search with the stated tie rule.
"""
import numpy as np
import pytest
import torch

from oracle import formats as F


def _all_bf16_as_f32(positive_only=False):
    bits = np.arange(1 << 16, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    ok = np.isfinite(v)
    if positive_only:
        ok &= v > 0
    return v[ok]


def _neighbours(vals64):
    """binary32 values at and within +-2 ulp of each of the given (exact) points."""
    v = np.asarray(vals64, dtype=np.float32)
    out = [v]
    up, dn = v.copy(), v.copy()
    for _ in range(2):
        up = np.nextafter(up, np.float32(np.inf))
        dn = np.nextafter(dn, np.float32(0))
        out += [up, dn]
    return np.concatenate(out)


# ------------------------------------------------------------------------------- E4M3
def test_e4m3_table_matches_torch_decode():
    codes = torch.arange(127, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(F.E4M3_POS, ref)
    assert F.E4M3_POS[-1] == 448.0 and F.E4M3_POS[1] == 2.0 ** -9


def test_e4m3_nearest_matches_torch_rne():
    mids = (F.E4M3_POS[:-1] + F.E4M3_POS[1:]) / 2
    x = np.concatenate([_all_bf16_as_f32(True), _neighbours(mids), _neighbours(F.E4M3_POS)])
    x = x[(x >= 0) & (x <= 448.0)]
    got = F.E4M3_POS[F.e4m3_nearest_code(x)]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(got, ref)


def test_e4m3_saturates():
    assert F.E4M3_POS[F.e4m3_nearest_code(np.float32([464.0, 1e30]))].tolist() == [448.0, 448.0]


# ------------------------------------------------------------------------------- E8M0
def test_e8m0_projection_matches_torch():
    ks = np.arange(-126, 127)
    pts = np.concatenate([2.0 ** ks, 1.5 * 2.0 ** ks[:-1]])
    x = np.concatenate([_all_bf16_as_f32(True), _neighbours(pts)])
    x = x[(x >= 2.0 ** -126) & (x < 1.5 * 2.0 ** 126)]
    got = np.ldexp(1.0, F.e8m0_nearest_exp(x))
    ref = torch.from_numpy(x).to(torch.float8_e8m0fnu).to(torch.float64).numpy()
    np.testing.assert_array_equal(got, ref)


def test_e8m0_projection_brute_force_and_clamp():
    rng = np.random.default_rng(1)
    x = np.concatenate([np.exp(rng.uniform(-95, 95, 4000)), [1.5, 3.0, 0.75, 1.4999999]])
    x = x.astype(np.float32)
    x = x[np.isfinite(x) & (x > 0)]
    pows = 2.0 ** np.arange(F.E8M0_KMIN, F.E8M0_KMAX + 1)
    d = np.abs(x.astype(np.float64)[:, None] - pows[None, :])
    best = d.min(axis=1, keepdims=True)
    # nearest; on an exact tie the larger power of two
    ref = np.array([pows[np.nonzero(row == b)[0].max()] for row, b in zip(d, best[:, 0])])
    got = np.ldexp(1.0, F.e8m0_nearest_exp(x))
    np.testing.assert_array_equal(got, ref)
    assert F.e8m0_nearest_exp(np.float32([1.5]))[0] == 1
    assert F.e8m0_nearest_exp(np.float32([3e38]))[0] == 127
    assert F.e8m0_nearest_exp(np.float32([1e-44]))[0] == -127


# ------------------------------------------------------------------------------- bf16
def test_bf16_nearest_matches_torch():
    rng = np.random.default_rng(2)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(0.01),
        np.exp(rng.uniform(-80, 80, 100000)).astype(np.float32),
    ])
    # exact ties: bf16 value + half a bf16 ulp
    b = (x.view(np.uint32) & np.uint32(0xFFFF0000))
    ties = (b | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties])
    x = x[np.isfinite(x)]
    got = F.bf16_nearest_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, ref)


# ------------------------------------------------------------------------------- E2M1
def _e2m1_value_from_bits(code):
    s, e, m = code >> 3, (code >> 1) & 3, code & 1
    mag = m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return -mag if s else mag


def test_e2m1_table_matches_bit_definition():
    for code in range(16):
        assert F.decode_elem(np.array([code]), F.make_format("MXFP4"))[0] == \
            _e2m1_value_from_bits(code)
    assert F.E2M1_MAG.tolist() == [_e2m1_value_from_bits(c) for c in range(8)]


def _brute_round(x, grid_codes, value_of):
    """Nearest grid value by exhaustive search; exact ties to the even code."""
    out = []
    for xv in np.asarray(x, dtype=np.float64):
        best = None
        for code in grid_codes:
            v = value_of(code)
            d = abs(xv - v)
            key = (d, code % 2)           # smaller distance, then even code
            if best is None or key < best[0]:
                best = (key, code, v)
        out.append(best[2])
    return np.array(out)


@pytest.mark.parametrize("kind", ["MXFP4", "NVFP4"])
def test_e2m1_round_brute_force(kind):
    fmt = F.make_format(kind)
    rng = np.random.default_rng(3)
    mids = (F.E2M1_MAG[:-1] + F.E2M1_MAG[1:]) / 2
    x = np.concatenate([rng.uniform(-8, 8, 3000), _neighbours(mids), -_neighbours(mids),
                        _neighbours(F.E2M1_MAG[1:]), [7.0, 100.0, -100.0]]).astype(np.float32)
    _, got = F.round_elem(x, fmt)
    mags = _brute_round(np.abs(x), range(8), _e2m1_value_from_bits)
    np.testing.assert_array_equal(np.abs(got), mags)
    assert np.all(np.signbit(got) == np.signbit(x))


@pytest.mark.parametrize("kind", ["MXFP4", "MXINT4"])
def test_element_rounding_saturates_for_huge_inputs(kind):
    fmt = F.make_format(kind)
    x = np.float32([1e6, 7.3e16, 1e30, 3.4e38, -7.3e16, -3.4e38])
    _, q = F.round_elem(x, fmt)
    top = fmt.qmax
    assert q.tolist() == [top] * 4 + [-top, -top]
    assert F.E4M3_POS[F.e4m3_nearest_code(np.float32([7.3e16, 3.4e38]))].tolist() == [448.0] * 2


def test_e2m1_documented_ties():
    fmt = F.make_format("MXFP4")
    x = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, -0.25, -5.0])
    _, q = F.round_elem(x, fmt)
    assert q.tolist() == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, -0.0, -4.0]


def test_int4_round_brute_force():
    fmt = F.make_format("INT4")
    rng = np.random.default_rng(4)
    x = np.concatenate([rng.uniform(-9, 9, 3000), np.arange(-8, 8) + 0.5]).astype(np.float32)
    _, got = F.round_elem(x, fmt)
    ref = _brute_round(x, range(-7, 8), float)
    np.testing.assert_array_equal(got, ref)


def test_int4_codes_are_twos_complement():
    fmt = F.make_format("MXINT4")
    codes, q = F.round_elem(np.float32([-7, -1, 0, 1, 7, -9, 9]), fmt)
    assert codes.tolist() == [9, 15, 0, 1, 7, 9, 7]
    np.testing.assert_array_equal(F.decode_elem(codes, fmt), q)


def test_int8_round_matches_torch_and_brute_force():
    """INT8 elements (the 8-bit appendix table): RNE onto -127..127, saturating; torch's
    round (half to even) and clamp, and the nearest-integer brute force, agree."""
    for kind in ("INT8", "MXINT8"):
        fmt = F.make_format(kind)
        rng = np.random.default_rng(6)
        x = np.concatenate([rng.uniform(-140, 140, 4000), np.arange(-130, 130) + 0.5,
                            [127.5, -127.5, 128.0, -128.0, 1e30, -1e30]]).astype(np.float32)
        codes, got = F.round_elem(x, fmt)
        ref_t = torch.clamp(torch.round(torch.from_numpy(x).double()), -127, 127).numpy()
        np.testing.assert_array_equal(got, ref_t)
        np.testing.assert_array_equal(got[:3000], _brute_round(x[:3000], range(-127, 128), float))
        # codes are the two's-complement bytes of the integers (torch's int8 view)
        tb = torch.from_numpy(got.astype(np.int8)).view(torch.uint8).numpy()
        np.testing.assert_array_equal(codes, tb)
        np.testing.assert_array_equal(F.decode_elem(codes, fmt), got)
        assert 0x80 not in set(codes.tolist())          # -128 is never produced


def test_int8_codes_are_stored_one_per_byte():
    codes = np.arange(256, dtype=np.uint8).reshape(4, 64)
    np.testing.assert_array_equal(F.pack_codes(codes, 8), codes)
    np.testing.assert_array_equal(F.unpack_codes(F.pack_codes(codes, 8), 8), codes)


def test_pack_roundtrip_low_nibble_even_column():
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 16, (3, 8)).astype(np.uint8)
    p = F.pack_codes(codes)
    assert p[0, 0] == (codes[0, 0] | (codes[0, 1] << 4))
    np.testing.assert_array_equal(F.unpack_codes(p), codes)


# --------------------------------------------------------------------- scale projection
def test_nvfp4_projection_is_nearest_in_linear_distance():
    fmt = F.make_format("NVFP4")
    s_t = F.nvfp4_tensor_scale(0.3)
    rng = np.random.default_rng(6)
    v = (np.exp(rng.uniform(-12, 6, 5000)) * float(s_t)).astype(np.float32)
    codes, val = F.project_scale(v, fmt, s_t)
    cand = (np.float32(s_t) * F.E4M3_POS[1:].astype(np.float32)).astype(np.float64)
    d = np.abs(v.astype(np.float64)[:, None] - cand[None, :])
    best = cand[np.argmin(d, axis=1)]
    # the decision is taken on fl32(v / s_t); away from midpoints it is the exact nearest
    dmin = np.sort(d, axis=1)
    clear = (dmin[:, 1] - dmin[:, 0]) > 1e-5 * v
    np.testing.assert_array_equal(val.astype(np.float64)[clear], best[clear])
    assert np.all(codes >= 1)


def test_nvfp4_tensor_scale_is_correctly_rounded_division():
    for a in [0.3, 1.0, 448.0, 1e-20, 3.0e38]:
        st = F.nvfp4_tensor_scale(a)
        ref = torch.tensor([np.float32(a)], dtype=torch.float32) / torch.tensor([2688.0])
        assert np.float32(st) == np.float32(ref.item())
    assert F.nvfp4_tensor_scale(0.0) == np.float32(1.0)


def test_int4_scale_clamps_to_min_normal():
    fmt = F.make_format("INT4")
    codes, val = F.project_scale(np.float32([1e-40, 0.0, 1.0]), fmt)
    assert codes.tolist() == [0x0080, 0x0080, 0x3F80]
