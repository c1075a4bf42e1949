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
// Layout of the work: the launch holds as many warps as the SMs keep resident; each warp owns
// a strip of 512 channels and an equal share of the token rows (a contiguous range), each
// lane a chunk of 16 consecutive channels of the strip (bf16: two 16-byte loads); a lane
// keeps its 16 column scales in registers for all its rows and walks down the rows, so a
// warp's loads, its 8-byte code stores and its scale stores are contiguous and c is read
// once per warp. A block of B channels spans B/16 lanes, which combine their absolute maxima
// with xor shuffles; the block scale (two correctly rounded divisions and a reciprocal) is
// computed once per 16 elements. The quantization pass loads the next row's chunk before it
// works on the current one. NVFP4 needs the global amax of x~ first (a separate pass that
// keeps AMAX_UNROLL rows of chunks in flight per lane; X is usually still in L2 for the
// second read).
#include <algorithm>

#include "dq_device.cuh"
#include "dq_internal.h"

namespace dq {
namespace {

constexpr unsigned FULL = 0xFFFFFFFFu;
constexpr int ACT_WARPS = 8;
constexpr int CHUNK = 16;                 // channels per lane and round
constexpr int AMAX_UNROLL = 4;            // chunks per lane in flight in the amax pass
constexpr int STRIP = CHUNK * 32;         // channels of one warp's strip

// 16 channels as raw words (bf16: 8 words; fp32: 16 words)
template <bool F32IN>
struct Chunk {
  uint32_t u[F32IN ? 16 : 8];
};

template <bool F32IN>
__device__ __forceinline__ void load_chunk(const void* X, int64_t row, int64_t ldx,
                                           int64_t col, Chunk<F32IN>& d) {
  if constexpr (F32IN) {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(X) +
                                                    row * ldx + col);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const uint4 v = __ldg(p + h);
      d.u[4 * h] = v.x; d.u[4 * h + 1] = v.y; d.u[4 * h + 2] = v.z; d.u[4 * h + 3] = v.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(X) +
                                                    row * ldx + col);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 v = __ldg(p + h);
      d.u[4 * h] = v.x; d.u[4 * h + 1] = v.y; d.u[4 * h + 2] = v.z; d.u[4 * h + 3] = v.w;
    }
  }
}

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

__device__ __forceinline__ float absmax16(const float2 (&x)[8]) {
  float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    a0 = max_nan(a0, fabsf(x[p].x));
    a1 = max_nan(a1, fabsf(x[p].y));
  }
  return max_nan(a0, a1);
}

// Warp -> (strip, row range): strip = warp % strips; the wps warps of a strip split the
// rows evenly (ranges differ by at most one row)
struct WarpWork {
  int64_t col, row0, row1;
};
__device__ __forceinline__ WarpWork warp_work(const ActLaunch& A, int64_t wps, int strips) {
  const int64_t w = (int64_t)blockIdx.x * ACT_WARPS + threadIdx.x / 32;
  const int64_t k = w / strips;
  WarpWork ww;
  ww.col = (int64_t)(w % strips) * STRIP + CHUNK * (threadIdx.x & 31);
  ww.row0 = (k < wps) ? (k * A.tokens) / wps : A.tokens;
  ww.row1 = (k < wps) ? ((k + 1) * A.tokens) / wps : A.tokens;
  return ww;
}

template <bool F32IN>
__global__ void act_amax_kernel(const ActLaunch A, const int64_t wps, const int strips) {
  const int lane = threadIdx.x & 31;
  const WarpWork ww = warp_work(A, wps, strips);
  const int64_t col = ww.col, row0 = ww.row0, row1 = ww.row1;
  const bool valid = col < A.n;
  float2 cv[8];
  load_c16(A.c, col, valid, cv);
  float a = 0.0f;
  // AMAX_UNROLL rows per step, all their loads issued before any use (no stores here)
  for (int64_t r0 = row0; r0 < row1; r0 += AMAX_UNROLL) {
    Chunk<F32IN> d[AMAX_UNROLL];
#pragma unroll
    for (int u = 0; u < AMAX_UNROLL; ++u) {
      if (valid && r0 + u < row1) load_chunk<F32IN>(A.X, r0 + u, A.ldx, col, d[u]);
      else zero_chunk<F32IN>(d[u]);
    }
#pragma unroll
    for (int u = 0; u < AMAX_UNROLL; ++u) {
      float2 x[8];
      rescale_chunk<F32IN>(d[u], cv, x);
      a = max_nan(a, absmax16(x));
    }
  }
  const bool bad = !isfinite(a);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(FULL, a, off));
  // one atomic per CTA: the maxima of its warps meet in shared memory first (every warp of
  // the launch updating one word serialises at its L2 slice)
  __shared__ float wmax[ACT_WARPS];
  if (lane == 0) wmax[threadIdx.x / 32] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.0f;
#pragma unroll
    for (int w = 0; w < ACT_WARPS; ++w) m = fmaxf(m, wmax[w]);
    if (m > 0.0f) atomicMax(A.amax_bits, __float_as_uint(m));
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

template <int ELEM, int SCALE, int B, bool F32IN>
__global__ void __launch_bounds__(ACT_WARPS * 32, 3)
act_quant_kernel(const ActLaunch A, const int64_t wps, const int strips) {
  constexpr int LB = B / CHUNK;                   // lanes per block
  constexpr float QMAX = elem_qmax<ELEM>();
  constexpr int SCB = (SCALE == SCALE_BF16) ? 2 : 1;
  constexpr bool BYTE_CODES = (ELEM == ELEM_INT8);         // one code byte per element
  const int lane = threadIdx.x & 31;
  const WarpWork ww = warp_work(A, wps, strips);
  const int64_t col = ww.col, row0 = ww.row0, row1 = ww.row1;
  const bool valid = col < A.n;
  float s_t = 1.0f;
  // NVFP4: every E4M3 code's decoded scale fl32(s_t * e) and its reciprocal, per CTA
  __shared__ float2 tbl[SCALE == SCALE_E4M3 ? 128 : 1];
  if constexpr (SCALE == SCALE_E4M3) {
    s_t = nvfp4_tensor_scale(__uint_as_float(*A.amax_bits));
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
  Chunk<F32IN> nxt;
  if (valid && row0 < row1) load_chunk<F32IN>(A.X, row0, A.ldx, col, nxt);
  else zero_chunk<F32IN>(nxt);
  for (int64_t row = row0; row < row1; ++row) {
    const Chunk<F32IN> cur = nxt;
    // the next row's chunk is in flight while this one is quantized
    if (valid && row + 1 < row1) load_chunk<F32IN>(A.X, row + 1, A.ldx, col, nxt);
    float2 x[8];
    rescale_chunk<F32IN>(cur, cv, x);
    float a = absmax16(x);
    bad |= !isfinite(a);
#pragma unroll
    for (int off = 1; off < LB; off <<= 1) a = max_nan(a, __shfl_xor_sync(FULL, a, off));
    uint32_t code = 0;
    float inv = 0.0f;
    if (a > 0.0f) {
      const ScaleVal sv = project_scale<SCALE>(__fdiv_rn(a, QMAX), s_t, tbl);
      code = sv.code;
      inv = sv.ir;
    }
    const float2 iv = make_float2(inv, inv);
    uint32_t w[4] = {0u, 0u, 0u, 0u};
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
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        float2 q;
        const uint32_t cb = quant2<ELEM>(mul2(x[p], iv), q);
        if constexpr (BYTE_CODES) w[p >> 1] |= (cb & 0xFFFFu) << (16 * (p & 1));
        else w[p >> 2] |= (cb & 0xFFu) << (8 * (p & 3));
      }
    }
    if (valid) {
      if (a == 0.0f) w[0] = w[1] = w[2] = w[3] = 0u;   // all-zero block: code 0 (also -0)
      if constexpr (BYTE_CODES) {
        uint8_t* dst = A.x_packed + row * qpitch + col;
        if (wide) {
          *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
          reinterpret_cast<uint2*>(dst)[0] = make_uint2(w[0], w[1]);
          reinterpret_cast<uint2*>(dst)[1] = make_uint2(w[2], w[3]);
        }
      } else {
        uint8_t* dst = A.x_packed + row * qpitch + col / 2;
        if (wide) {
          *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
        } else {
          reinterpret_cast<uint32_t*>(dst)[0] = w[0];
          reinterpret_cast<uint32_t*>(dst)[1] = w[1];
        }
      }
      if ((lane % LB) == 0) {
        const int64_t b = col / B;
        if constexpr (SCB == 2) {
          reinterpret_cast<uint16_t*>(A.scales)[row * nb + b] = (uint16_t)code;
        } else if constexpr (SCALE == SCALE_E4M3) {
          // the W4A4 GEMM's layout: [row / 128][n / 64][512 bytes], the four scales of a
          // 64-channel group of row r at (r % 32) * 16 + (r % 128 / 32) * 4
          const int64_t r = row & 127;
          const int64_t off = A.sf_tc ? ((row >> 7) * (A.n / 64) + (b >> 2)) * 512 +
                                            (r & 31) * 16 + (r >> 5) * 4 + (b & 3)
                                      : row * nb + b;
          reinterpret_cast<uint8_t*>(A.scales)[off] = (uint8_t)code;
        } else {
          reinterpret_cast<uint8_t*>(A.scales)[row * nb + b] = (uint8_t)code;
        }
      }
    }
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

// launch over (strips x wps) warps: at most the resident warps, at least one row each
template <auto KERNEL>
cudaError_t launch_rows(const ActLaunch& A, cudaStream_t s) {
  const int strips = (int)((A.n + STRIP - 1) / STRIP);
  const int64_t wps = std::max<int64_t>(1, std::min<int64_t>(resident_warps<KERNEL>() / strips,
                                                             A.tokens));
  const int64_t ctas = (wps * strips + ACT_WARPS - 1) / ACT_WARPS;
  KERNEL<<<(unsigned)ctas, ACT_WARPS * 32, 0, s>>>(A, wps, strips);
  count_launches(1);
  return cudaGetLastError();
}

template <int ELEM, int SCALE, int B>
cudaError_t launch_fmt(const ActLaunch& A, int esize, cudaStream_t s) {
  if (SCALE == SCALE_E4M3) {
    const cudaError_t e = (esize == 4) ? launch_rows<act_amax_kernel<true>>(A, s)
                                       : launch_rows<act_amax_kernel<false>>(A, s);
    if (e != cudaSuccess) return e;
  }
  return (esize == 4) ? launch_rows<act_quant_kernel<ELEM, SCALE, B, true>>(A, s)
                      : launch_rows<act_quant_kernel<ELEM, SCALE, B, false>>(A, s);
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
