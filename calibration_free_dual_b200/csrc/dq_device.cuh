// dq_device.cuh — device-side codecs and projections shared by the DualQuant kernels.
//
// Element grids: INT4 (-7..7), INT8 (-127..127) and E2M1 (OCP MX v1.0 FP4); block scales:
// bf16, E8M0 and
// E4M3 (FN) times an fp32 tensor scale. Every rounding is round-to-nearest-even on a binary32
// input (E8M0: nearest power of two, tie up), saturating at the grid's largest magnitude.
// Pi_S maps a scale to the nearest member of the format's set of representable block
// scales: the projection step that the DualQuant abstract (acceptodds.com/papers/
// iclr2027-49818) applies after every scale update.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace dq {

enum Elem : int { ELEM_INT4 = 0, ELEM_E2M1 = 1, ELEM_INT8 = 2 };

// largest element magnitude of a grid
template <int ELEM>
__host__ __device__ constexpr float elem_qmax() {
  return ELEM == ELEM_INT4 ? 7.0f : (ELEM == ELEM_INT8 ? 127.0f : 6.0f);
}
enum Scale : int { SCALE_BF16 = 0, SCALE_E8M0 = 1, SCALE_E4M3 = 2 };

// error bits of the per-device error word
constexpr unsigned ERRBIT_NONFINITE = 1u;
constexpr unsigned ERRBIT_TIMEOUT = 2u;
constexpr unsigned ERRBIT_BADWARM = 4u;

constexpr float NVFP4_TENSOR_DIV = 2688.0f;   // 6 (E2M1 max) * 448 (E4M3 max)

// ------------------------------------------------------------------ bf16 <-> fp32 (exact)
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// ------------------------------------------------------------------ E2M1 elements
// Two binary32 values -> one byte of two E2M1 codes (low nibble = lo), RNE, saturating.
__device__ __forceinline__ uint32_t e2m1x2_encode(float lo, float hi) {
  uint16_t out;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\tmov.b16 %0, {t, 0};\n\t}"
      : "=h"(out) : "f"(lo), "f"(hi));
  return out;
}
// One byte of two E2M1 codes -> their values (low nibble -> .x).
__device__ __forceinline__ float2 e2m1x2_decode(uint32_t byte) {
  uint32_t h2;
  uint16_t b = (uint16_t)(byte & 0xFFu);
  asm("{\n\t.reg .b8 t, tz;\n\tmov.b16 {t, tz}, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(h2) : "h"(b));
  __half2 hv = *reinterpret_cast<__half2*>(&h2);
  return __half22float2(hv);
}

// ------------------------------------------------------------------ INT4 / INT8 elements
__device__ __forceinline__ float int4_round(float x) {
  return fminf(fmaxf(rintf(x), -7.0f), 7.0f);
}
__device__ __forceinline__ uint32_t int4_code(float q) { return ((int)q) & 0xF; }
__device__ __forceinline__ float int8_round(float x) {
  return fminf(fmaxf(rintf(x), -127.0f), 127.0f);
}
__device__ __forceinline__ uint32_t int8_code(float q) { return ((int)q) & 0xFF; }

// Quantize a pair on the element grid: values into q; codes of x.x and x.y, x.x lowest:
// one byte of two nibbles (4-bit grids) or two bytes (INT8).
template <int ELEM>
__device__ __forceinline__ uint32_t quant2(float2 x, float2& q) {
  if constexpr (ELEM == ELEM_E2M1) {
    uint32_t code = e2m1x2_encode(x.x, x.y);
    q = e2m1x2_decode(code);
    return code;
  } else if constexpr (ELEM == ELEM_INT8) {
    q.x = int8_round(x.x);
    q.y = int8_round(x.y);
    return int8_code(q.x) | (int8_code(q.y) << 8);
  } else {
    q.x = int4_round(x.x);
    q.y = int4_round(x.y);
    return int4_code(q.x) | (int4_code(q.y) << 4);
  }
}

// Quantized values of a pair only (no code): E2M1 encode and decode in one step, the code
// never leaves the conversion unit's 8-bit register.
template <int ELEM>
__device__ __forceinline__ float2 quant2_value(float2 x) {
  if constexpr (ELEM == ELEM_E2M1) {
    uint32_t h2;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(h2) : "f"(x.x), "f"(x.y));
    __half2 hv = *reinterpret_cast<__half2*>(&h2);
    return __half22float2(hv);
  } else if constexpr (ELEM == ELEM_INT8) {
    return make_float2(int8_round(x.x), int8_round(x.y));
  } else {
    return make_float2(int4_round(x.x), int4_round(x.y));
  }
}

// ------------------------------------------------------------------ E4M3 (FN)
// Nearest E4M3 code of u >= 0 (RNE, saturating at 448); code 0 for u that rounds to 0.
__device__ __forceinline__ uint32_t e4m3_encode(float u) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(u));
  return out & 0xFFu;
}
__device__ __forceinline__ float e4m3_decode(uint32_t code) {
  uint32_t h2;
  uint16_t b = (uint16_t)(code & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(b));
  __half2 hv = *reinterpret_cast<__half2*>(&h2);
  return __low2float(hv);
}

// ------------------------------------------------------------------ E8M0
// Exact 2^k for k in [-149, 127].
__device__ __forceinline__ float pow2_exact(int k) {
  return (k >= -126) ? __uint_as_float((uint32_t)(k + 127) << 23)
                     : __uint_as_float(1u << (k + 149));
}
// Code k+127 of the power of two nearest to v (tie at 1.5*2^k goes up), k in [-127, 127];
// v <= 0 (only reachable through underflow) gives the smallest, 2^-127.
__device__ __forceinline__ uint32_t e8m0_encode(float v) {
  if (!(v > 0.0f)) return 0u;
  uint32_t b = __float_as_uint(v);
  int E = (int)(b >> 23);
  uint32_t M = b & 0x7FFFFFu;
  int k;
  if (E == 0) {
    k = (M >= 0x600000u) ? -126 : -127;   // subnormal: nearest of 2^-127, 2^-126
  } else if (E == 255) {
    k = 127;
  } else {
    k = E - 127 + (M >= 0x400000u ? 1 : 0);
  }
  k = max(-127, min(127, k));
  return (uint32_t)(k + 127);
}
__device__ __forceinline__ float e8m0_decode(uint32_t code) { return pow2_exact((int)code - 127); }

// ------------------------------------------------------------------ bf16 scale
__device__ __forceinline__ uint32_t bf16_rn_bits(float v) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// ------------------------------------------------------------------ projection Pi_S
struct ScaleVal {
  float r;        // decoded scale
  float ir;       // fl32(1 / r)
  uint32_t code;  // stored code
};

// Decode a stored scale code. `tbl` (E4M3 only) holds fl32(s_t*e) and fl32(1/that) per code.
template <int SCALE>
__device__ __forceinline__ ScaleVal scale_decode(uint32_t code, const float2* tbl) {
  ScaleVal s;
  s.code = code;
  if constexpr (SCALE == SCALE_BF16) {
    s.r = __uint_as_float(code << 16);
    s.ir = __frcp_rn(s.r);
  } else if constexpr (SCALE == SCALE_E8M0) {
    s.r = pow2_exact((int)code - 127);
    s.ir = pow2_exact(127 - (int)code);
  } else {
    float2 t = tbl[code];
    s.r = t.x;
    s.ir = t.y;
  }
  return s;
}

// A bf16 block scale from its code with 1/r from a table of the 128 mantissa reciprocals
// rtab[f] = fl32(1 / (1 + f/128)): for a normal code with exponent field E <= 252, fl32(1/r)
// is rtab[f] * 2^(127 - E) exactly (a power-of-two scaling that stays in the normal range),
// formed by adding to the exponent bits; the two largest binades (a subnormal reciprocal)
// take the correctly rounded reciprocal.
__device__ __forceinline__ ScaleVal bf16_scale_decode_tab(uint32_t code, const float* rtab) {
  ScaleVal s;
  s.code = code;
  s.r = __uint_as_float(code << 16);
  const uint32_t E = (code >> 7) & 0xFFu;
  s.ir = (E <= 252u) ? __uint_as_float(__float_as_uint(rtab[code & 0x7Fu]) + ((127u - E) << 23))
                     : __frcp_rn(s.r);
  return s;
}

// fl32(num / den) for binary64 num >= 0, den > 0 (normal), by a reciprocal: the hardware's
// approximate binary64 reciprocal refined by two Newton-Raphson steps y <- y + y(1 - den y)
// (each squares the relative error), so that num * y is within a few binary64 ulps of the
// quotient before its rounding to binary32. It can differ from fl32 of the correctly rounded
// binary64 quotient only within a few binary64 ulps of a binary32 midpoint, far inside the
// rounding of the binary64 sums num and den themselves.
__device__ __forceinline__ float div64_to_f32(double num, double den) {
  double y;
  asm("rcp.approx.ftz.f64 %0, %1;" : "=d"(y) : "d"(den));
  double e = fma(-den, y, 1.0);
  y = fma(y, e, y);
  e = fma(-den, y, 1.0);
  y = fma(y, e, y);
  return __double2float_rn(num * y);
}

// Nearest admissible scale to v (binary32), as a code: bf16 RNE clamped to [2^-126, max];
// E8M0 nearest power of two; E4M3: e = RNE(fl32(v / s_t)) raised to 2^-9 if 0 (the scale is
// then fl32(s_t * e)).
template <int SCALE>
__device__ __forceinline__ uint32_t project_code(float v, float s_t) {
  uint32_t code;
  if constexpr (SCALE == SCALE_BF16) {
    code = (v > 0.0f) ? bf16_rn_bits(v) : 0x0080u;
    code = min(max(code, 0x0080u), 0x7F7Fu);
  } else if constexpr (SCALE == SCALE_E8M0) {
    code = e8m0_encode(v);
  } else {
    float u = (v > 0.0f) ? __fdiv_rn(v, s_t) : 0.0f;
    code = max(e4m3_encode(u), 1u);
  }
  return code;
}

// The same projection, decoded.
template <int SCALE>
__device__ __forceinline__ ScaleVal project_scale(float v, float s_t, const float2* tbl) {
  return scale_decode<SCALE>(project_code<SCALE>(v, s_t), tbl);
}

// Projection of the least-squares scale num/den inside a BCD iteration. The quotient is a
// binary32 approximation (its summands are binary32 sums already): fast division, and for
// E4M3 the scaled quotient num / (den * s_t) directly. An empty block (den = 0: every code
// of the block is 0) keeps `old_code`; the code is selected first and decoded once, with no
// branch around the projection.
template <int SCALE>
__device__ __forceinline__ ScaleVal project_scale_ls(float num, float den, float s_t,
                                                     const float2* tbl, uint32_t old_code) {
  uint32_t code;
  if constexpr (SCALE == SCALE_BF16) {
    const float v = __fdividef(num, den);
    code = (v > 0.0f) ? bf16_rn_bits(v) : 0x0080u;
    code = min(max(code, 0x0080u), 0x7F7Fu);
  } else if constexpr (SCALE == SCALE_E8M0) {
    code = e8m0_encode(__fdividef(num, den));
  } else {
    // num >= +0 (every w*q >= 0: q has the sign of w) and den > 0, so u >= +0; the high
    // half of the conversion is the code of +0, so the low byte is the whole result
    const float u = __fdividef(num, __fmul_rn(den, s_t));
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(u));
    code = max((uint32_t)(out & 0xFFu), 1u);
  }
  code = (den > 0.0f) ? code : old_code;
  return scale_decode<SCALE>(code, tbl);
}

// Same projection without the per-CTA E4M3 table (decoded scale computed directly).
template <int SCALE>
__device__ __forceinline__ ScaleVal project_scale_direct(float v, float s_t) {
  if constexpr (SCALE == SCALE_E4M3) {
    const float u = (v > 0.0f) ? __fdiv_rn(v, s_t) : 0.0f;
    ScaleVal sv;
    sv.code = max(e4m3_encode(u), 1u);
    sv.r = __fmul_rn(s_t, e4m3_decode(sv.code));
    sv.ir = __frcp_rn(sv.r);
    return sv;
  } else {
    return project_scale<SCALE>(v, s_t, nullptr);
  }
}

// Correctly rounded a / Q for the grid maxima Q = 6, 7, 127 and finite a >= 0, in three
// operations: q0 = fl32(a * y) with y = fl32(1/Q), the exact residual r = a - q0*Q by one
// fma, and q1 = fl32(q0 + r*y) by another (the one-step correction of P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990). Checked against binary64 division over every positive binary32: exact
// for Q = 7 and 127, and for Q = 6 whenever a >= 2^-125; below that (quotients in the
// subnormal range) the IEEE division is used.
template <int Q>
__device__ __forceinline__ float div_qmax(float a) {
  static_assert(Q == 6 || Q == 7 || Q == 127, "verified divisors only");
  constexpr float y = 1.0f / (float)Q;
  if (Q == 6 && a < 0x1p-125f) return __fdiv_rn(a, (float)Q);
  const float q0 = __fmul_rn(a, y);
  const float r = __fmaf_rn(-q0, (float)Q, a);
  return __fmaf_rn(r, y, q0);
}

// NVFP4 per-tensor scale from the amax bit pattern.
__device__ __forceinline__ float nvfp4_tensor_scale(float amax) {
  return (amax > 0.0f) ? __fdiv_rn(amax, NVFP4_TENSOR_DIV) : 1.0f;
}

// max that propagates NaN (a NaN operand gives NaN): a running |x| maximum is non-finite
// exactly when one of its inputs is, so one test per block or row piece suffices
__device__ __forceinline__ float max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// ------------------------------------------------------------------ packed fp32x2 math
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

}  // namespace dq
