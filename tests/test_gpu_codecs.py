"""Bit-exact parity of the device codecs with the oracle's tables (B200)."""
import numpy as np
import pytest
import torch

from oracle import formats as F

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dq():
    import calibration_free_dual_b200 as pkg
    return pkg


def _bf16_all():
    bits = np.arange(1 << 16, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    return v[np.isfinite(v)]


def _near(points, k=3):
    v = np.asarray(points, dtype=np.float32)
    out = [v]
    up, dn = v.copy(), v.copy()
    for _ in range(k):
        up = np.nextafter(up, np.float32(np.inf))
        dn = np.nextafter(dn, np.float32(-np.inf))
        out += [up, dn]
    return np.concatenate(out)


def _run_encode(dq, x, codec):
    xt = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    return dq.encode(xt, codec).cpu().numpy()


def test_e2m1_encode_bit_exact(dq):
    mids = (F.E2M1_MAG[:-1] + F.E2M1_MAG[1:]) / 2
    x = np.concatenate([_bf16_all(), _near(mids), -_near(mids), _near(F.E2M1_MAG),
                        np.random.default_rng(0).uniform(-8, 8, 200000).astype(np.float32)])
    got = _run_encode(dq, x, dq.DQ_CODEC_E2M1)
    ref, _ = F.round_elem(x, F.make_format("MXFP4"))
    mism = np.nonzero(got != ref)[0]
    assert mism.size == 0, (x[mism[:10]], got[mism[:10]], ref[mism[:10]])


def test_int4_encode_bit_exact(dq):
    x = np.concatenate([_bf16_all(), _near(np.arange(-8, 8) + 0.5),
                        np.random.default_rng(1).uniform(-9, 9, 200000).astype(np.float32)])
    got = _run_encode(dq, x, dq.DQ_CODEC_INT4)
    ref, _ = F.round_elem(x, F.make_format("INT4"))
    np.testing.assert_array_equal(got, ref)


def test_int8_encode_bit_exact(dq):
    x = np.concatenate([_bf16_all(), _near(np.arange(-130, 130) + 0.5),
                        np.random.default_rng(2).uniform(-140, 140, 200000).astype(np.float32)])
    got = _run_encode(dq, x, dq.DQ_CODEC_INT8)
    ref, _ = F.round_elem(x, F.make_format("INT8"))
    np.testing.assert_array_equal(got, ref)


def test_e4m3_encode_bit_exact(dq):
    mids = (F.E4M3_POS[:-1] + F.E4M3_POS[1:]) / 2
    x = np.concatenate([_bf16_all(), _near(mids), _near(F.E4M3_POS), [500.0, 1e30]])
    x = np.abs(x[np.isfinite(x)]).astype(np.float32)
    got = _run_encode(dq, x, dq.DQ_CODEC_E4M3)
    ref = F.e4m3_nearest_code(x)
    np.testing.assert_array_equal(got.astype(np.int64), ref)


def test_e8m0_encode_bit_exact(dq):
    ks = np.arange(-126, 127)
    pts = np.concatenate([2.0 ** ks, 1.5 * 2.0 ** ks[:-1], [1.5 * 2.0 ** -127, 2.0 ** -127]])
    x = np.concatenate([_bf16_all(), _near(pts)]).astype(np.float32)
    x = x[np.isfinite(x) & (x > 0)]
    got = _run_encode(dq, x, dq.DQ_CODEC_E8M0).astype(np.int64)
    ref = F.e8m0_nearest_exp(x) + 127
    np.testing.assert_array_equal(got, ref)


def test_bf16_encode_bit_exact(dq):
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(300000).astype(np.float32) * np.float32(0.02),
                        np.exp(rng.uniform(-80, 80, 100000)).astype(np.float32)])
    ties = ((x.view(np.uint32) & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties])
    x = x[np.isfinite(x)]
    got = _run_encode(dq, x, dq.DQ_CODEC_BF16).view(np.uint16)
    np.testing.assert_array_equal(got, F.bf16_nearest_bits(x))


@pytest.mark.parametrize("codec,kind,ncodes", [(1, "MXFP4", 16), (0, "MXINT4", 16),
                                              (5, "MXINT8", 256)])
def test_element_decode_all_codes(dq, codec, kind, ncodes):
    codes = torch.arange(ncodes, dtype=torch.uint8).cuda()
    got = dq.decode(codes, codec).cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(got, F.decode_elem(np.arange(ncodes), F.make_format(kind)))


def test_scale_decode_all_codes(dq):
    e4 = dq.decode(torch.arange(127, dtype=torch.uint8).cuda(), dq.DQ_CODEC_E4M3).cpu().numpy()
    np.testing.assert_array_equal(e4.astype(np.float64), F.E4M3_POS)
    e8 = dq.decode(torch.arange(255, dtype=torch.uint8).cuda(), dq.DQ_CODEC_E8M0).cpu().numpy()
    np.testing.assert_array_equal(e8.astype(np.float64), 2.0 ** (np.arange(255) - 127))
