// dq_act.cu — activation rescale by the solver's column scales + block quantization (4-bit
// formats; INT8 and MXINT8 for the appendix's 8-bit W8A8 setting).
//
// DualQuant ("DualQuant: Dual-scale Calibration-free Weight-and-Activation Quantization for
// LLMs", Abstract; appendix Table 11, activation quantization including beta; appendix
// Table 6, activation SQNR with and without beta): the column scales of the weight solve
// rescale the activation channels before a 4-bit block quantizer, with no calibration
// data. With W_hat = diag(r) Q diag(c) the quantized GEMM consumes c * x, so the kernel
// quantizes x~ = fl32(X * c).
//
// Layout of the work: each warp owns a strip of 512 channels and a contiguous range of token
// rows (rows per warp set on the host so that the launch holds about as many warps as the SMs
// keep resident); each lane owns a chunk of 16 consecutive channels of the strip, keeps its
// 16 column scales in registers for all its rows and walks down the rows, so a warp's loads,
// its 8-byte code stores and its scale stores are contiguous and c is read once per warp.
// Rows arrive through a per-lane ring of asynchronous copies in shared memory (several rows
// in flight, no registers held); the quantization pass works on two rows at a time (two
// independent chains). A block of B channels spans B/16 lanes, which combine their
// absolute maxima with xor shuffles; the block scale is computed once per 16 elements. NVFP4
// needs the global amax of x~ first: a separate pass over the same rows that writes one
// maximum per CTA (no atomics, nothing to clear beforehand); the quantization pass is launched
// as its programmatic dependent, so its launch overlaps the pre-pass, and it reduces those
// maxima itself once the pre-pass has completed (X is usually still in L2 for its second
// read).
#include <algorithm>

#include "dq_device.cuh"
#include "dq_internal.h"

namespace dq {
namespace {

constexpr unsigned FULL = 0xFFFFFFFFu;
constexpr int ACT_WARPS = 8;
constexpr int CHUNK = 16;                 // channels per lane and round
constexpr int STRIP = CHUNK * 32;         // channels of one warp's strip

// 16 channels as raw words (bf16: 8 words; fp32: 16 words)
template <bool F32IN>
struct Chunk {
  uint32_t u[F32IN ? 16 : 8];
};

// A lane's copy-ahead ring in shared memory: its chunks of the next RD rows are in flight as
// asynchronous copies (no registers held) while it works on the current row. Every lane
// copies and reads only its own slots, so no lane waits on another. Chunk h of lane l sits
// at l*CB + (h ^ swizzle(l)), which spreads a quarter warp's 16-byte reads over all banks.
template <bool F32IN, int RD>
struct LaneRing {
  static constexpr int CB = F32IN ? 4 : 2;          // 16-byte chunks per lane and row
  uint4* base;                                      // this warp's [RD][32 * CB] slots
  int lane, sw;
  __device__ __forceinline__ LaneRing(uint4* warp_base, int l)
      : base(warp_base), lane(l), sw(CB == 2 ? ((l >> 2) & 1) : ((l >> 1) & 3)) {}
  // the lane's chunk at `src` (when `in`) into slot `slot`; one commit group per call
  __device__ __forceinline__ void issue(const char* src, bool in, int slot) const {
    if (in) {
      const uint32_t dst = static_cast<uint32_t>(
          __cvta_generic_to_shared(base + (size_t)slot * 32 * CB + lane * CB));
#pragma unroll
      for (int h = 0; h < CB; ++h)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;"
                     :: "r"(dst + 16u * (uint32_t)(h ^ sw)), "l"(src + 16 * h) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  // the chunk of the oldest pending row, in slot `slot`, once its copy has landed
  __device__ __forceinline__ void read(int slot, Chunk<F32IN>& d) const {
    asm volatile("cp.async.wait_group %0;" :: "n"(RD - 1) : "memory");
    const uint4* q = base + (size_t)slot * 32 * CB + lane * CB;
#pragma unroll
    for (int h = 0; h < CB; ++h) {
      const uint4 v = q[h ^ sw];
      d.u[4 * h] = v.x; d.u[4 * h + 1] = v.y; d.u[4 * h + 2] = v.z; d.u[4 * h + 3] = v.w;
    }
  }
};
constexpr int AMAX_RING = 5;              // rows in flight per lane, amax pass
constexpr int QUANT_RING = 5;             // rows in flight per lane, quantization pass

template <bool F32IN>
__device__ __forceinline__ void zero_chunk(Chunk<F32IN>& d) {
#pragma unroll
  for (int i = 0; i < (F32IN ? 16 : 8); ++i) d.u[i] = 0u;
}

// the chunk's 16 column scales (1 without c or past the last channel)
__device__ __forceinline__ void load_c16(const float* c, int64_t col, bool valid,
                                         float2 (&cv)[8]) {
  if (c == nullptr || !valid) {
#pragma unroll
    for (int p = 0; p < 8; ++p) cv[p] = make_float2(1.0f, 1.0f);
    return;
  }
  const float4* cp = reinterpret_cast<const float4*>(c + col);
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const float4 v = __ldg(cp + h);
    cv[2 * h] = make_float2(v.x, v.y);
    cv[2 * h + 1] = make_float2(v.z, v.w);
  }
}

// x~ = fl32(X * c) of the chunk, as 8 pairs (multiplying by 1 is exact: X itself without c)
template <bool F32IN>
__device__ __forceinline__ void rescale_chunk(const Chunk<F32IN>& d, const float2 (&cv)[8],
                                              float2 (&x)[8]) {
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    if constexpr (F32IN) x[p] = make_float2(__uint_as_float(d.u[2 * p]), __uint_as_float(d.u[2 * p + 1]));
    else x[p] = bf16x2_to_f2(d.u[p]);
    x[p] = mul2(x[p], cv[p]);
  }
}

// Warp -> (strip, row range): strip = warp % strips; warp k of a strip takes rows
// [k * rpw, (k + 1) * rpw) clipped to the tokens (rpw: rows per warp, from the host)
struct WarpWork {
  int64_t col, row0, row1;
};
__device__ __forceinline__ WarpWork warp_work(const ActLaunch& A, int64_t rpw, int strips) {
  const unsigned w = blockIdx.x * ACT_WARPS + threadIdx.x / 32;
  const unsigned k = w / (unsigned)strips;
  WarpWork ww;
  ww.col = (int64_t)(w - k * (unsigned)strips) * STRIP + CHUNK * (threadIdx.x & 31);
  ww.row0 = min((int64_t)k * rpw, A.tokens);
  ww.row1 = min(ww.row0 + rpw, A.tokens);
  return ww;
}

// largest |x| of a chunk (NaN if any is NaN), two independent chains
__device__ __forceinline__ float absmax16(const float2 (&x)[8]) {
  float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    a0 = max_nan(a0, fabsf(x[p].x));
    a1 = max_nan(a1, fabsf(x[p].y));
  }
  return max_nan(a0, a1);
}

template <bool F32IN>
__global__ void act_amax_kernel(const ActLaunch A, const int64_t rpw, const int strips) {
  // the quantization pass may start launching now; it waits for this grid's completion
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const WarpWork ww = warp_work(A, rpw, strips);
  const int64_t col = ww.col, row0 = ww.row0, row1 = ww.row1;
  const bool valid = col < A.n;
  float2 cv[8];
  load_c16(A.c, col, valid, cv);
  float a = 0.0f;
  constexpr int RD = F32IN ? AMAX_RING / 2 : AMAX_RING;
  __shared__ __align__(16) uint4 ring_mem[ACT_WARPS][RD * 32 * LaneRing<F32IN, RD>::CB];
  const LaneRing<F32IN, RD> ring(ring_mem[threadIdx.x / 32], lane);
  const int64_t step = A.ldx * (F32IN ? 4 : 2);
  const char* src = reinterpret_cast<const char*>(A.X) + (row0 * A.ldx + col) * (F32IN ? 4 : 2);
#pragma unroll
  for (int j = 0; j < RD; ++j) {
    ring.issue(src, valid && row0 + j < row1, j);
    src += step;
  }
  int slot = 0;
  for (int64_t row = row0; row < row1; ++row) {
    Chunk<F32IN> d;
    ring.read(slot, d);
    if (!valid) zero_chunk<F32IN>(d);       // a lane past the last channel copied nothing
    float2 x[8];
    rescale_chunk<F32IN>(d, cv, x);        // the chunk is in registers: its slot is free
    ring.issue(src, valid && row + RD < row1, slot);
    src += step;
    a = max_nan(a, absmax16(x));
    slot = (slot + 1 == RD) ? 0 : slot + 1;
  }
  const bool bad = !isfinite(a);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(FULL, a, off));
  // one maximum per CTA, written to its own slot (the quantization pass reduces them)
  __shared__ float wmax[ACT_WARPS];
  if (lane == 0) wmax[threadIdx.x / 32] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.0f;
#pragma unroll
    for (int w = 0; w < ACT_WARPS; ++w) m = fmaxf(m, wmax[w]);
    A.partials[blockIdx.x] = __float_as_uint(m);
  }
  if (bad) atomicOr(A.err_word, ERRBIT_NONFINITE);
}

// Eight binary32 values -> one word of eight E2M1 codes (RNE, saturating), value k in
// nibble k (byte k/2, low nibble first)
__device__ __forceinline__ uint32_t e2m1x8_encode(const float2 (&y)[4]) {
  uint32_t out;
  asm("{\n\t.reg .b8 t0, t1, t2, t3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t3, %8, %7;\n\t"
      "mov.b32 %0, {t0, t1, t2, t3};\n\t}"
      : "=r"(out)
      : "f"(y[0].x), "f"(y[0].y), "f"(y[1].x), "f"(y[1].y), "f"(y[2].x), "f"(y[2].y),
        "f"(y[3].x), "f"(y[3].y));
  return out;
}

// The quantized codes of one 16-channel chunk on an integer grid (INT4 -7..7, INT8
// -127..127): y = fl32(x * inv) clamped to [-Q, Q], then rounded to the nearest integer
// (ties to even) by adding 1.5 * 2^23, whose last byte is then the integer's two's
// complement. INT4: eight nibbles per word (value k in nibble k); INT8: four bytes per word.
//
// With a bf16 block scale s = bf16(fl32(a / Q)) (a the block's largest |x|), |x| / s stays
// below Q / (1 - 2^-8) < Q + 1/2 (bf16 rounds with relative error at most 2^-8, and the binary32
// roundings of 1/s and of the product move it by under 2^-22 relative), so the rounded code is
// within [-Q, Q] without the clamp; CLAMP is needed for the E8M0 scales (a power of two can sit
// up to a factor of 2 below a / Q).
template <int ELEM, bool CLAMP>
__device__ __forceinline__ void int_codes(const float2 (&x)[8], float2 iv, uint32_t (&w)[4]) {
  constexpr float Q = elem_qmax<ELEM>();
  const float2 magic = make_float2(12582912.0f, 12582912.0f), one = make_float2(1.0f, 1.0f);
  uint32_t b[16];
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    float2 y = mul2(x[p], iv);
    if constexpr (CLAMP) {
      y.x = fminf(fmaxf(y.x, -Q), Q);
      y.y = fminf(fmaxf(y.y, -Q), Q);
    }
    const float2 z = fma2(y, one, magic);
    b[2 * p] = __float_as_uint(z.x);
    b[2 * p + 1] = __float_as_uint(z.y);
  }
  if constexpr (ELEM == ELEM_INT8) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      w[k] = __byte_perm(__byte_perm(b[4 * k], b[4 * k + 1], 0x0040),
                         __byte_perm(b[4 * k + 2], b[4 * k + 3], 0x0040), 0x5410);
  } else {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      uint32_t by[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        // byte j: nibble of value 2j in the low half, of value 2j+1 in the high half
        const uint32_t lo = b[8 * k + 2 * j], hi = b[8 * k + 2 * j + 1] << 4;
        by[j] = (lo & 0x0Fu) | (hi & 0xF0u);
      }
      w[k] = __byte_perm(__byte_perm(by[0], by[1], 0x0040), __byte_perm(by[2], by[3], 0x0040),
                         0x5410);
    }
  }
}

template <int ELEM, int SCALE, int B, bool F32IN, bool SF_TC>
__global__ void __launch_bounds__(ACT_WARPS * 32, 2)
act_quant_kernel(const ActLaunch A, const int64_t rpw, const int strips, const int nparts) {
  constexpr int LB = B / CHUNK;                   // lanes per block
  constexpr float QMAX = elem_qmax<ELEM>();
  constexpr int SCB = (SCALE == SCALE_BF16) ? 2 : 1;
  constexpr bool BYTE_CODES = (ELEM == ELEM_INT8);         // one code byte per element
  const int lane = threadIdx.x & 31;
  const WarpWork ww = warp_work(A, rpw, strips);
  const int64_t col = ww.col, row0 = ww.row0, row1 = ww.row1;
  const bool valid = col < A.n;
  float s_t = 1.0f, is_t = 1.0f;
  // NVFP4: every E4M3 code's decoded scale fl32(s_t * e) and its reciprocal, per CTA
  __shared__ float2 tbl[SCALE == SCALE_E4M3 ? 128 : 1];
  if constexpr (SCALE == SCALE_E4M3) {
    // the pre-pass (this grid's programmatic predecessor) has completed and its maxima are
    // visible after the wait; every CTA reduces them (a few KB from L2)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ uint32_t pmax[ACT_WARPS];
    uint32_t mx = 0u;
    for (int i = threadIdx.x; i < nparts; i += blockDim.x) mx = max(mx, A.partials[i]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) mx = max(mx, __shfl_xor_sync(FULL, mx, off));
    if ((threadIdx.x & 31) == 0) pmax[threadIdx.x / 32] = mx;
    __syncthreads();
    mx = 0u;
#pragma unroll
    for (int w = 0; w < ACT_WARPS; ++w) mx = max(mx, pmax[w]);
    s_t = nvfp4_tensor_scale(__uint_as_float(mx));
    is_t = __frcp_rn(s_t);
    if (blockIdx.x == 0 && threadIdx.x == 0 && A.tensor_scale != nullptr) *A.tensor_scale = s_t;
    if (threadIdx.x < 128) {
      const uint32_t code = (threadIdx.x == 0 || threadIdx.x == 127) ? 1u : threadIdx.x;
      const float r = __fmul_rn(s_t, e4m3_decode(code));
      tbl[threadIdx.x] = make_float2(r, __frcp_rn(r));
    }
    __syncthreads();
  }
  const int64_t nb = A.n / B, qpitch = BYTE_CODES ? A.n : A.n / 2;
  // a lane's codes (8 bytes; 16 for the 8-bit formats) go out in one store when the code
  // buffer's base allows it (row pitches and chunk offsets are multiples of that size)
  const bool wide = (reinterpret_cast<uintptr_t>(A.x_packed) & (BYTE_CODES ? 15u : 7u)) == 0;
  float2 cv[8];
  load_c16(A.c, col, valid, cv);
  bool bad = false;
  constexpr int RD = F32IN ? QUANT_RING / 2 : QUANT_RING;
  __shared__ __align__(16) uint4 ring_mem[ACT_WARPS][RD * 32 * LaneRing<F32IN, RD>::CB];
  const LaneRing<F32IN, RD> ring(ring_mem[threadIdx.x / 32], lane);
  // running addresses: the next row to copy, the code and scale destinations of this row
  const int64_t step = A.ldx * (F32IN ? 4 : 2);
  const char* src = reinterpret_cast<const char*>(A.X) + (row0 * A.ldx + col) * (F32IN ? 4 : 2);
#pragma unroll
  for (int j = 0; j < RD; ++j) {
    ring.issue(src, valid && row0 + j < row1, j);
    src += step;
  }
  uint8_t* qdst = A.x_packed + row0 * qpitch + (BYTE_CODES ? col : col / 2);
  const int64_t b = col / B;
  int64_t sidx = row0 * nb + b;
  int slot = 0;
  // one row's chunk from the ring (the next row of the lane's range is then put in flight)
  auto load_row = [&](int64_t row, float2 (&x)[8]) {
    // (a lane past the last channel copied nothing and computes on stale values: its block
    // lies wholly past the last channel, and nothing of it is stored or flagged)
    Chunk<F32IN> cur;
    ring.read(slot, cur);
    rescale_chunk<F32IN>(cur, cv, x);      // the chunk is in registers: its slot is free
    ring.issue(src, valid && row + RD < row1, slot);
    src += step;
    slot = (slot + 1 == RD) ? 0 : slot + 1;
  };
  // the block maximum, scale code, reciprocal and element codes of one row
  auto quant_row = [&](const float2 (&x)[8], float& a, uint32_t& code, uint32_t (&w)[4]) {
    a = absmax16(x);
    // (NVFP4: the pre-pass has flagged any non-finite x~ already)
    if constexpr (SCALE != SCALE_E4M3) bad |= valid && !isfinite(a);
#pragma unroll
    for (int off = 1; off < LB; off <<= 1) a = max_nan(a, __shfl_xor_sync(FULL, a, off));
    code = 0;
    float inv = 0.0f;
    if (a > 0.0f) {
      const float v = div_qmax<(int)QMAX>(a);
      if constexpr (SCALE == SCALE_E4M3) {
        // E4M3 of fl32(v / s_t) through the reciprocal: v * fl32(1/s_t) lies within 3 ulps of
        // the quotient, and E4M3 rounds (in its normal range) at the binary32 patterns whose
        // low 20 bits are 0x80000; a product in [2^-6, 448) farther than 8 ulps from one
        // rounds as the quotient does, anything else takes the division
        const float u1 = v * is_t;
        const uint32_t lo = __float_as_uint(u1) & 0xFFFFFu;
        code = (u1 >= 0x1p-6f && u1 < 448.0f && (lo + 8u - 0x80000u) > 16u)
                   ? e4m3_encode(u1) : project_code<SCALE>(v, s_t);
        inv = tbl[code].y;
      } else {
        const ScaleVal sv = project_scale<SCALE>(v, s_t, tbl);
        code = sv.code;
        inv = sv.ir;
      }
    }
    const float2 iv = make_float2(inv, inv);
    w[0] = w[1] = w[2] = w[3] = 0u;
    if constexpr (ELEM == ELEM_E2M1) {
      // four conversions straight into the bytes of one word
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float2 y[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) y[k] = mul2(x[4 * h + k], iv);
        w[h] = e2m1x8_encode(y);
      }
    } else {
      int_codes<ELEM, SCALE != SCALE_BF16>(x, iv, w);
    }
  };
  // the row's codes and scale code (blocks of a lane past the last channel: nothing)
  auto store_row = [&](int64_t row, uint8_t* qdst, int64_t sidx, float a, uint32_t code,
                       uint32_t (&w)[4]) {
    if (valid) {
      if (a == 0.0f) w[0] = w[1] = w[2] = w[3] = 0u;   // all-zero block: code 0 (also -0)
      if constexpr (BYTE_CODES) {
        if (wide) {
          *reinterpret_cast<uint4*>(qdst) = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
          reinterpret_cast<uint2*>(qdst)[0] = make_uint2(w[0], w[1]);
          reinterpret_cast<uint2*>(qdst)[1] = make_uint2(w[2], w[3]);
        }
      } else {
        if (wide) {
          *reinterpret_cast<uint2*>(qdst) = make_uint2(w[0], w[1]);
        } else {
          reinterpret_cast<uint32_t*>(qdst)[0] = w[0];
          reinterpret_cast<uint32_t*>(qdst)[1] = w[1];
        }
      }
      if ((lane % LB) == 0) {
        if constexpr (SCB == 2) {
          reinterpret_cast<uint16_t*>(A.scales)[sidx] = (uint16_t)code;
        } else if constexpr (SCALE == SCALE_E4M3) {
          // the W4A4 GEMM's layout: [row / 128][n / 64][512 bytes], the four scales of a
          // 64-channel group of row r at (r % 32) * 16 + (r % 128 / 32) * 4
          int64_t off = sidx;
          if constexpr (SF_TC) {
            const int64_t r = row & 127;
            off = ((row >> 7) * (A.n / 64) + (b >> 2)) * 512 + (r & 31) * 16 + (r >> 5) * 4 +
                  (b & 3);
          }
          reinterpret_cast<uint8_t*>(A.scales)[off] = (uint8_t)code;
        } else {
          reinterpret_cast<uint8_t*>(A.scales)[sidx] = (uint8_t)code;
        }
      }
    }
  };
  // two rows per iteration: two independent chains for the scheduler to interleave
  int64_t row = row0;
  for (; row + 1 < row1; row += 2, qdst += 2 * qpitch, sidx += 2 * nb) {
    float2 x0[8], x1[8];
    load_row(row, x0);
    load_row(row + 1, x1);
    float a0, a1;
    uint32_t c0, c1, w0[4], w1[4];
    quant_row(x0, a0, c0, w0);
    quant_row(x1, a1, c1, w1);
    store_row(row, qdst, sidx, a0, c0, w0);
    store_row(row + 1, qdst + qpitch, sidx + nb, a1, c1, w1);
  }
  if (row < row1) {
    float2 x0[8];
    load_row(row, x0);
    float a0;
    uint32_t c0, w0[4];
    quant_row(x0, a0, c0, w0);
    store_row(row, qdst, sidx, a0, c0, w0);
  }
  if (bad) atomicOr(A.err_word, ERRBIT_NONFINITE);
}

// Warps the SMs keep resident for a kernel (queried once per kernel and process, with a
// thread-safe static; a failed query falls back to one CTA per SM of a 148-SM part).
template <auto KERNEL>
int64_t resident_warps() {
  static const int64_t warps = [] {
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, KERNEL, ACT_WARPS * 32, 0) !=
            cudaSuccess)
      return (int64_t)148 * ACT_WARPS;
    return (int64_t)std::max(sms, 1) * std::max(per_sm, 1) * ACT_WARPS;
  }();
  return warps;
}

// The grid of a pass: (strips x warps per strip), at most the resident warps (and cap_ctas
// CTAs); rows per warp rpw = ceil(tokens / warps per strip), and only the warps with rows
// are launched.
struct RowGrid {
  int strips;
  int64_t rpw, ctas;
};
template <auto KERNEL>
RowGrid row_grid(const ActLaunch& A, int64_t cap_ctas) {
  RowGrid g;
  g.strips = (int)((A.n + STRIP - 1) / STRIP);
  const int64_t warps = std::min<int64_t>(resident_warps<KERNEL>(), cap_ctas * ACT_WARPS);
  const int64_t wps = std::max<int64_t>(1, std::min<int64_t>(warps / g.strips, A.tokens));
  g.rpw = std::max<int64_t>(1, (A.tokens + wps - 1) / wps);
  const int64_t used = std::max<int64_t>(1, (A.tokens + g.rpw - 1) / g.rpw);
  g.ctas = (used * g.strips + ACT_WARPS - 1) / ACT_WARPS;
  return g;
}

template <int ELEM, int SCALE, int B, bool F32IN, bool SF_TC>
cudaError_t launch_fmt_dt(const ActLaunch& A, cudaStream_t s) {
  constexpr auto QK = act_quant_kernel<ELEM, SCALE, B, F32IN, SF_TC>;
  const RowGrid gq = row_grid<QK>(A, INT64_MAX / ACT_WARPS);
  if constexpr (SCALE != SCALE_E4M3) {
    QK<<<(unsigned)gq.ctas, ACT_WARPS * 32, 0, s>>>(A, gq.rpw, gq.strips, 0);
    count_launches(1);
    return cudaGetLastError();
  } else {
    constexpr auto AK = act_amax_kernel<F32IN>;
    const RowGrid ga = row_grid<AK>(A, ACT_MAX_PARTS);
    AK<<<(unsigned)ga.ctas, ACT_WARPS * 32, 0, s>>>(A, ga.rpw, ga.strips);
    count_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)gq.ctas);
    cfg.blockDim = dim3(ACT_WARPS * 32);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, QK, A, gq.rpw, gq.strips, (int)ga.ctas);
    count_launches(1);
    return e;
  }
}

// the tensor core's scale layout exists for NVFP4 only
template <int ELEM, int SCALE, int B, bool F32IN>
cudaError_t launch_layout(const ActLaunch& A, cudaStream_t s) {
  if constexpr (SCALE == SCALE_E4M3) {
    if (A.sf_tc) return launch_fmt_dt<ELEM, SCALE, B, F32IN, true>(A, s);
  }
  return launch_fmt_dt<ELEM, SCALE, B, F32IN, false>(A, s);
}

template <int ELEM, int SCALE, int B>
cudaError_t launch_fmt(const ActLaunch& A, int esize, cudaStream_t s) {
  return (esize == 4) ? launch_layout<ELEM, SCALE, B, true>(A, s)
                      : launch_layout<ELEM, SCALE, B, false>(A, s);
}

}  // namespace

cudaError_t launch_act(const ActLaunch& A, int kind, int group, int esize, cudaStream_t s) {
  switch (kind) {
    case 0:
      if (group == 64) return launch_fmt<ELEM_INT4, SCALE_BF16, 64>(A, esize, s);
      return launch_fmt<ELEM_INT4, SCALE_BF16, 128>(A, esize, s);
    case 1: return launch_fmt<ELEM_INT4, SCALE_E8M0, 32>(A, esize, s);
    case 2: return launch_fmt<ELEM_E2M1, SCALE_E8M0, 32>(A, esize, s);
    case 3: return launch_fmt<ELEM_E2M1, SCALE_E4M3, 16>(A, esize, s);
    case 4:
      if (group == 64) return launch_fmt<ELEM_INT8, SCALE_BF16, 64>(A, esize, s);
      return launch_fmt<ELEM_INT8, SCALE_BF16, 128>(A, esize, s);
    case 5: return launch_fmt<ELEM_INT8, SCALE_E8M0, 32>(A, esize, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dq
