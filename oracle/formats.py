"""Element grids and block-scale sets as explicit value tables (oracle; test only).

The DualQuant pages name the formats (INT4 grouped, MXINT4, MXFP4, NVFP4 with E4M3 block
scales and an FP32 tensor scale; the 8-bit appendix table: INT8 G=128 and MXINT8 G=32) but
not their bit layouts; the tables below follow the
public OCP Microscaling v1.0 definitions (E2M1 elements, E8M0 scales) and the usual FP8
E4M3 ("FN": no infinities, 0x7F is NaN) definition. Every rounding is "nearest value in the
table", with the tie rule stated beside it, computed in binary64 on a binary32 input, so the
decision is exact for that binary32 value.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

# --- element grids ---------------------------------------------------------------------
# E2M1 magnitudes by 3-bit code (exponent bits 2..1 with bias 1, mantissa bit 0).
E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])

# E4M3 non-negative values by code 0..126 (code 127 is NaN): exponent bits 6..3, bias 7,
# mantissa bits 2..0; exponent 0 is subnormal (m * 2^-9).
def _e4m3_value(code: int) -> float:
    e, mt = code >> 3, code & 7
    if e == 0:
        return mt * 2.0 ** -9
    return (1.0 + mt / 8.0) * 2.0 ** (e - 7)


E4M3_POS = np.array([_e4m3_value(c) for c in range(127)])
E4M3_MAX = 448.0
E4M3_MIN_POS = 2.0 ** -9

BF16_MIN_NORMAL_BITS = 0x0080       # 2^-126
BF16_MAX_BITS = 0x7F7F              # largest finite bf16
E8M0_KMIN, E8M0_KMAX = -127, 127
NVFP4_TENSOR_DIV = 6.0 * 448.0      # E2M1 max times E4M3 max

FORMAT_KINDS = ("INT4", "MXINT4", "MXFP4", "NVFP4", "INT8", "MXINT8")


@dataclass(frozen=True)
class Format:
    kind: str
    block: int

    @property
    def elem(self) -> str:
        return {"INT4": "int4", "MXINT4": "int4", "MXFP4": "e2m1", "NVFP4": "e2m1",
                "INT8": "int8", "MXINT8": "int8"}[self.kind]

    @property
    def scale(self) -> str:
        return {"INT4": "bf16", "MXINT4": "e8m0", "MXFP4": "e8m0", "NVFP4": "e4m3",
                "INT8": "bf16", "MXINT8": "e8m0"}[self.kind]

    @property
    def qmax(self) -> float:
        return {"int4": 7.0, "e2m1": 6.0, "int8": 127.0}[self.elem]

    @property
    def bits(self) -> int:
        """Bits per element code: 4 (two codes per byte) or 8 (one byte, two's complement)."""
        return 8 if self.elem == "int8" else 4


def make_format(kind: str, block: int | None = None) -> Format:
    """The formats by name; `block` overrides the block length (tests use tiny blocks)."""
    default = {"INT4": 128, "MXINT4": 32, "MXFP4": 32, "NVFP4": 16, "INT8": 128,
               "MXINT8": 32}[kind]
    return Format(kind, int(block if block is not None else default))


# --- element rounding ------------------------------------------------------------------
def _nearest_sorted(vals: np.ndarray, x: np.ndarray) -> np.ndarray:
    """Index of the nearest entry of the ascending table `vals` to each x (x >= 0).

    Exact ties go to the even index (the even code); beyond the last entry the last
    entry is returned (saturation)."""
    x = np.asarray(x, dtype=np.float64)
    hi = np.searchsorted(vals, x, side="left")
    hi = np.clip(hi, 0, len(vals) - 1)
    lo = np.clip(hi - 1, 0, len(vals) - 1)
    d_lo = np.abs(x - vals[lo])
    d_hi = np.abs(vals[hi] - x)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    # saturation, stated directly: far beyond the table the binary64 distances to the last
    # two entries can round to the same value
    return np.where(x >= vals[-1], len(vals) - 1, idx)


def round_elem(x32: np.ndarray, fmt: Format):
    """RNE of binary32 x onto the element grid, saturating.

    Returns (codes uint8, values float64). INT4 codes are two's-complement nibbles of the
    integer, INT8 codes its two's-complement byte (symmetric grid -127..127, like INT4's
    -7..7: the most negative code is never produced); E2M1 codes are sign<<3 | magnitude
    code, the sign taken from x's sign bit."""
    x = np.asarray(x32, dtype=np.float32).astype(np.float64)
    if fmt.elem in ("int4", "int8"):
        qm = fmt.qmax
        q = np.clip(np.rint(x), -qm, qm)             # np.rint rounds half to even
        mask = 0xF if fmt.elem == "int4" else 0xFF
        codes = (q.astype(np.int64) & mask).astype(np.uint8)
        return codes, q
    neg = np.signbit(x)
    idx = _nearest_sorted(E2M1_MAG, np.abs(x))
    mag = E2M1_MAG[idx]
    codes = (idx + 8 * neg).astype(np.uint8)
    return codes, np.where(neg, -mag, mag)


def decode_elem(codes: np.ndarray, fmt: Format) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.int64)
    if fmt.elem == "int4":
        return np.where(codes >= 8, codes - 16, codes).astype(np.float64)
    if fmt.elem == "int8":
        return np.where(codes >= 128, codes - 256, codes).astype(np.float64)
    mag = E2M1_MAG[codes & 7]
    return np.where(codes & 8, -mag, mag)


# --- scale projection ------------------------------------------------------------------
def bf16_nearest_bits(v32: np.ndarray) -> np.ndarray:
    """Nearest bfloat16 (ties to even) to binary32 v, as uint16 bit patterns (finite v)."""
    bits = np.asarray(v32, dtype=np.float32).view(np.uint32).astype(np.int64)
    lo = bits & 0xFFFF0000
    hi = lo + 0x10000
    v = np.asarray(v32, dtype=np.float32).astype(np.float64)
    vlo = lo.astype(np.uint32).view(np.float32).astype(np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        vhi = hi.astype(np.uint32).view(np.float32).astype(np.float64)
        d_lo, d_hi = np.abs(v - vlo), np.abs(vhi - v)
    lo_even = ((lo >> 16) & 1) == 0
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ~lo_even)
    return (np.where(pick_hi, hi, lo) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32)


def e8m0_nearest_exp(v32: np.ndarray) -> np.ndarray:
    """Exponent k of the power of two nearest to v > 0 (tie at 1.5*2^k goes up), clamped."""
    v = np.asarray(v32, dtype=np.float32).astype(np.float64)
    mant, e = np.frexp(v)                 # v = mant * 2^e, mant in [0.5, 1)
    k = e - 1                             # v = (2*mant) * 2^k, 2*mant in [1, 2)
    k = k + (2.0 * mant >= 1.5)
    k = np.where(v > 0.0, k, E8M0_KMIN)  # a zero quotient (underflow) takes the smallest
    return np.clip(k, E8M0_KMIN, E8M0_KMAX).astype(np.int64)


def e4m3_nearest_code(u32: np.ndarray) -> np.ndarray:
    """Nearest non-negative E4M3 code to binary32 u >= 0 (ties to even code, saturating)."""
    return _nearest_sorted(E4M3_POS, np.asarray(u32, dtype=np.float32)).astype(np.int64)


def nvfp4_tensor_scale(amax: float) -> np.float32:
    """s_t = fl32(amax / (6*448)), or 1 when amax is 0."""
    if amax <= 0.0:
        return np.float32(1.0)
    return np.float32(np.float64(np.float32(amax)) / NVFP4_TENSOR_DIV)


def project_scale(v32: np.ndarray, fmt: Format, s_t: np.float32 | None = None):
    """Pi_S: nearest admissible block scale to binary32 v (v <= 0 gives the smallest).

    Returns (codes, decoded binary32 values). Codes: bf16 bits (INT4), k+127 (E8M0),
    E4M3 code (NVFP4; decoded value fl32(s_t * e))."""
    v32 = np.asarray(v32, dtype=np.float32)
    if fmt.scale == "bf16":
        b = bf16_nearest_bits(np.abs(v32)).astype(np.int64)
        b = np.where(v32 > 0, b, BF16_MIN_NORMAL_BITS)     # v <= 0: the smallest scale
        b = np.clip(b, BF16_MIN_NORMAL_BITS, BF16_MAX_BITS).astype(np.uint16)
        return b, bf16_bits_to_f32(b)
    if fmt.scale == "e8m0":
        k = e8m0_nearest_exp(v32)
        return (k + 127).astype(np.uint8), np.ldexp(np.float32(1.0), k).astype(np.float32)
    assert s_t is not None
    u = (v32 / np.float32(s_t)).astype(np.float32)           # binary32 quotient
    code = e4m3_nearest_code(u)
    code = np.maximum(code, 1)                                # no zero scale
    val = (np.float32(s_t) * E4M3_POS[code].astype(np.float32)).astype(np.float32)
    return code.astype(np.uint8), val


def decode_scale(codes: np.ndarray, fmt: Format, s_t: np.float32 | None = None):
    codes = np.asarray(codes)
    if fmt.scale == "bf16":
        return bf16_bits_to_f32(codes)
    if fmt.scale == "e8m0":
        return np.ldexp(np.float32(1.0), codes.astype(np.int64) - 127).astype(np.float32)
    return (np.float32(s_t) * E4M3_POS[codes.astype(np.int64)].astype(np.float32)).astype(
        np.float32)


def pack_codes(codes: np.ndarray, bits: int = 4) -> np.ndarray:
    """[rows, n] 4-bit codes -> [rows, n/2] bytes, low nibble = even column (8-bit codes
    are stored one per byte, unchanged)."""
    codes = np.asarray(codes, dtype=np.uint8)
    if bits == 8:
        return codes.copy()
    return (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)


def unpack_codes(packed: np.ndarray, bits: int = 4) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    if bits == 8:
        return packed.copy()
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out
