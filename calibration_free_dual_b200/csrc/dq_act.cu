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
// HBM-bound streaming kernel: one warp per token row; per round the 32 lanes cover 256
// consecutive channels, 8 per lane (one 16-byte load of bf16), so loads, the 4-byte code
// stores and the scale stores of a warp are contiguous. A block of B channels spans B/8
// lanes, which combine their absolute maxima with xor shuffles. NVFP4 needs the global
// amax of x~ first (a separate pass; X is usually still in L2 for the second read).
#include <algorithm>

#include "dq_device.cuh"
#include "dq_internal.h"

namespace dq {
namespace {

constexpr unsigned FULL = 0xFFFFFFFFu;
constexpr int ACT_WARPS = 8;

template <bool F32IN>
__device__ __forceinline__ void load8(const void* X, int64_t row, int64_t ldx, int64_t col,
                                      float (&x)[8]) {
  if constexpr (F32IN) {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(X) +
                                                      row * ldx + col);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(
        reinterpret_cast<const uint16_t*>(X) + row * ldx + col));
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = bf16x2_to_f2(u[k]);
      x[2 * k] = f.x;
      x[2 * k + 1] = f.y;
    }
  }
}

// max that propagates NaN (a NaN operand gives NaN): the running |x| maximum of a block is
// non-finite exactly when one of its elements is, so one test per block suffices
__device__ __forceinline__ float max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

__device__ __forceinline__ void rescale8(const float* c, int64_t col, float (&x)[8]) {
  if (c == nullptr) return;
  const float4 a = __ldg(reinterpret_cast<const float4*>(c + col));
  const float4 b = __ldg(reinterpret_cast<const float4*>(c + col) + 1);
  const float cv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 8; ++k) x[k] = __fmul_rn(x[k], cv[k]);
}

template <bool F32IN>
__global__ void act_amax_kernel(const ActLaunch A) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (int64_t)blockIdx.x * ACT_WARPS + threadIdx.x / 32;
  const int64_t nwarps = (int64_t)gridDim.x * ACT_WARPS;
  float a = 0.0f;
  for (int64_t row = warp0; row < A.tokens; row += nwarps) {
    for (int64_t col = 8 * lane; col < A.n; col += 256) {
      float x[8];
      load8<F32IN>(A.X, row, A.ldx, col, x);
      rescale8(A.c, col, x);
#pragma unroll
      for (int k = 0; k < 8; ++k) a = max_nan(a, fabsf(x[k]));
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

template <int ELEM, int SCALE, int B, bool F32IN>
__global__ void act_quant_kernel(const ActLaunch A) {
  constexpr int LB = B / 8;                       // lanes per block
  constexpr float QMAX = elem_qmax<ELEM>();
  constexpr int SCB = (SCALE == SCALE_BF16) ? 2 : 1;
  constexpr bool BYTE_CODES = (ELEM == ELEM_INT8);         // one code byte per element
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (int64_t)blockIdx.x * ACT_WARPS + threadIdx.x / 32;
  const int64_t nwarps = (int64_t)gridDim.x * ACT_WARPS;
  float s_t = 1.0f;
  if constexpr (SCALE == SCALE_E4M3) {
    s_t = nvfp4_tensor_scale(__uint_as_float(*A.amax_bits));
    if (blockIdx.x == 0 && threadIdx.x == 0 && A.tensor_scale != nullptr) *A.tensor_scale = s_t;
  }
  const int64_t nb = A.n / B, qpitch = BYTE_CODES ? A.n : A.n / 2;
  bool bad = false;
  for (int64_t row = warp0; row < A.tokens; row += nwarps) {
    for (int64_t base = 0; base < A.n; base += 256) {
      const int64_t col = base + 8 * lane;
      const bool valid = col < A.n;
      float x[8];
      if (valid) {
        load8<F32IN>(A.X, row, A.ldx, col, x);
        rescale8(A.c, col, x);
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = 0.0f;
      }
      float a = 0.0f;
#pragma unroll
      for (int k = 0; k < 8; ++k) a = max_nan(a, fabsf(x[k]));
      bad |= !isfinite(a);
#pragma unroll
      for (int off = 1; off < LB; off <<= 1) a = fmaxf(a, __shfl_xor_sync(FULL, a, off));
      uint32_t code = 0;
      float inv = 0.0f;
      if (a > 0.0f) {
        const ScaleVal sv = project_scale_direct<SCALE>(__fdiv_rn(a, QMAX), s_t);
        code = sv.code;
        inv = sv.ir;
      }
      uint64_t packed = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float2 q;
        uint32_t cb = quant2<ELEM>(make_float2(__fmul_rn(x[2 * k], inv), __fmul_rn(x[2 * k + 1], inv)), q);
        if constexpr (BYTE_CODES) packed |= (uint64_t)(cb & 0xFFFFu) << (16 * k);
        else packed |= (uint64_t)(cb & 0xFFu) << (8 * k);
      }
      if (valid) {
        if (a == 0.0f) packed = 0;   // all-zero block: code 0 (also for -0 inputs)
        if constexpr (BYTE_CODES)
          *reinterpret_cast<uint64_t*>(A.x_packed + row * qpitch + col) = packed;
        else
          *reinterpret_cast<uint32_t*>(A.x_packed + row * qpitch + col / 2) = (uint32_t)packed;
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
  }
  if (bad) atomicOr(A.err_word, ERRBIT_NONFINITE);
}

template <int ELEM, int SCALE, int B>
cudaError_t launch_fmt(const ActLaunch& A, int esize, cudaStream_t s) {
  const int64_t rows_per_cta = ACT_WARPS;
  int blocks = (int)std::min<int64_t>((A.tokens + rows_per_cta - 1) / rows_per_cta, 148 * 16);
  if (blocks < 1) blocks = 1;
  if (SCALE == SCALE_E4M3) {
    if (esize == 4) act_amax_kernel<true><<<blocks, ACT_WARPS * 32, 0, s>>>(A);
    else act_amax_kernel<false><<<blocks, ACT_WARPS * 32, 0, s>>>(A);
    count_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (esize == 4) act_quant_kernel<ELEM, SCALE, B, true><<<blocks, ACT_WARPS * 32, 0, s>>>(A);
  else act_quant_kernel<ELEM, SCALE, B, false><<<blocks, ACT_WARPS * 32, 0, s>>>(A);
  count_launches(1);
  return cudaGetLastError();
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
