"""Hand-worked activation quantization examples (tests/golden/worked_activations.txt).

The pages print no worked example; these were derived by hand from the activation path of
DualQuant (Abstract: the column scales rescale the activation channels before the 4-bit
quantizer; appendix Tables 6 and 11). They pin the oracle's rescale direction, block
maxima, scale projection (E4M3 with the tensor scale, bf16), zero blocks and element ties
with exact numbers (4-channel blocks on the CPU). The CUDA path is checked on the same numbers
with every block padded by zero channels to the format's real length.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import formats as F
from oracle.actquant import act_quant as ora_act

FIXTURE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                       "worked_activations.txt")
REAL_BLOCK = {"NVFP4": 16, "INT4": 128}


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
            key, val = (t.strip() for t in line.split(":", 1))
            rows = [r.split() for r in val.split("|")]
            if key == "fmt":
                cur[key] = val
            elif key == "codes":
                cur[key] = [[int(t, 16) for t in r] for r in rows]
            elif key == "scale_codes":
                cur[key] = [[int(t, 0) for t in r] for r in rows]
            elif key == "s_t":
                cur[key] = Fraction(val)
            else:
                cur[key] = [[Fraction(t) for t in r] for r in rows]
    return ex


EXAMPLES = _load()


def _f32(rows):
    return np.array([[float(v) for v in r] for r in rows], dtype=np.float32)


@pytest.mark.parametrize("name", sorted(EXAMPLES))
def test_oracle_reproduces_the_hand_example(name):
    ex = EXAMPLES[name]
    fmt = F.make_format(ex["fmt"], 4)
    out = ora_act(_f32(ex["X"]), fmt, _f32(ex["c"])[0])
    np.testing.assert_array_equal(out["codes"], np.array(ex["codes"], dtype=np.uint8))
    np.testing.assert_array_equal(out["scale_codes"].astype(np.int64),
                                  np.array(ex["scale_codes"], dtype=np.int64))
    if "s_t" in ex:
        assert out["s_t"] == np.float32(float(ex["s_t"]))


def _padded(ex):
    """Every 4-channel block padded with zero channels to the real block length."""
    B = REAL_BLOCK[ex["fmt"]]
    X = _f32(ex["X"])
    c = _f32(ex["c"])[0]
    T, n = X.shape
    nb = n // 4
    Xp = np.zeros((T, nb * B), dtype=np.float32)
    cp = np.ones(nb * B, dtype=np.float32)
    for b in range(nb):
        Xp[:, b * B:b * B + 4] = X[:, 4 * b:4 * b + 4]
        cp[b * B:b * B + 4] = c[4 * b:4 * b + 4]
    return Xp, cp, B


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(EXAMPLES))
def test_cuda_path_reproduces_the_hand_example(name):
    import torch
    import calibration_free_dual_b200 as dq

    ex = EXAMPLES[name]
    Xp, cp, B = _padded(ex)
    fmt = F.make_format(ex["fmt"], B)
    o = dq.act_quant(torch.from_numpy(Xp).cuda(), ex["fmt"], torch.from_numpy(cp).cuda())
    torch.cuda.synchronize()
    assert dq.last_device_error() == 0
    codes = F.unpack_codes(o["x_packed"].cpu().numpy(), fmt.bits)
    want = np.array(ex["codes"], dtype=np.uint8)
    T, n = want.shape
    for b in range(n // 4):
        np.testing.assert_array_equal(codes[:, b * B:b * B + 4], want[:, 4 * b:4 * b + 4])
        assert not codes[:, b * B + 4:(b + 1) * B].any()
    sc = o["scales"].cpu().numpy()
    sc = (sc.view(np.uint16) if fmt.scale == "bf16" else sc).astype(np.int64)
    np.testing.assert_array_equal(sc, np.array(ex["scale_codes"], dtype=np.int64))
    if "s_t" in ex:
        assert o["tensor_scale"].cpu().numpy()[0] == np.float32(float(ex["s_t"]))
