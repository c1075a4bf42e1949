// dq_solve.cu — host side of the solve (plan, launches), the NVFP4 amax pre-pass and the
// trace finalisation; the solve kernel itself is in dq_solve_kernel.cuh.
#include "dq_solve_kernel.cuh"

namespace dq {
namespace {

// ----------------------------------------------------------------------------- amax
// max |W| of every matrix (NVFP4 tensor scale): one warp per row, four 16-byte loads in
// flight per lane, maximum over the magnitude bits (for non-negative floats the bit patterns
// order like the values; a NaN counts as larger than any number, and the solve reports it).
template <int ESZ>
__device__ __forceinline__ uint32_t fold_abs(uint32_t mx, const uint4& v) {
  if constexpr (ESZ == 2) {
    mx = __vmaxu2(mx, v.x & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, v.y & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, v.z & 0x7FFF7FFFu);
    return __vmaxu2(mx, v.w & 0x7FFF7FFFu);
  } else {
    mx = max(mx, v.x & 0x7FFFFFFFu);
    mx = max(mx, v.y & 0x7FFFFFFFu);
    mx = max(mx, v.z & 0x7FFFFFFFu);
    return max(mx, v.w & 0x7FFFFFFFu);
  }
}

template <int ESZ>
__global__ void __launch_bounds__(256) solve_amax_kernel(const __grid_constant__ SolveLaunch L) {
  const SolveMat& M = L.mats[blockIdx.y];
  const int lane = threadIdx.x & 31;
  const int wid = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int nw = gridDim.x * (blockDim.x >> 5);
  const int cpr = L.n * ESZ / 16;                    // 16-byte chunks per row
  uint32_t mx = 0u;
  for (int row = wid; row < L.m; row += nw) {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(M.W) +
                                                    (int64_t)row * M.ldw * ESZ);
    int c = lane;
    for (; c + 96 < cpr; c += 128) {
      const uint4 v0 = ldg_stream(p + c), v1 = ldg_stream(p + c + 32);
      const uint4 v2 = ldg_stream(p + c + 64), v3 = ldg_stream(p + c + 96);
      mx = fold_abs<ESZ>(fold_abs<ESZ>(fold_abs<ESZ>(fold_abs<ESZ>(mx, v0), v1), v2), v3);
    }
    for (; c < cpr; c += 32) mx = fold_abs<ESZ>(mx, ldg_stream(p + c));
  }
  if constexpr (ESZ == 2) mx = max(mx & 0xFFFFu, mx >> 16) << 16;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) mx = max(mx, __shfl_xor_sync(FULL, mx, off));
  if (lane == 0 && mx != 0u) atomicMax(M.amax_bits, mx);
}

// ------------------------------------------------------------------------- finalize
struct FinalizeArgs {
  double* mse[SOLVE_MAXMATS];
  double* err[SOLVE_MAXMATS];
  double* wsq[SOLVE_MAXMATS];
  double* qout[SOLVE_MAXMATS];   // null: no Q-change trace
  double* qch[SOLVE_MAXMATS];
  int tiles[SOLVE_MAXMATS];
  int T;
};

__global__ void finalize_kernel(const __grid_constant__ FinalizeArgs A) {
  const int mat = blockIdx.y;
  const int t = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (t > A.T) return;
  const int tiles = A.tiles[mat];
  double e = 0.0, w = 0.0;
  for (int i = lane; i < tiles; i += 32) {
    e += A.err[mat][(int64_t)t * tiles + i];
    w += A.wsq[mat][i];
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    e += __shfl_xor_sync(FULL, e, off);
    w += __shfl_xor_sync(FULL, w, off);
  }
  if (lane == 0) A.mse[mat][t] = (w > 0.0) ? e / w : 0.0;
  if (A.qout[mat] != nullptr) {
    // sqrt(sum (q_t - q_{t-1})^2) / sqrt(sum q_{t-1}^2); both sums exact, so their order is free
    double d = 0.0, p = 0.0;
    if (t >= 2) {
      for (int i = lane; i < tiles; i += 32) {
        d += A.qch[mat][2 * ((int64_t)t * tiles + i)];
        p += A.qch[mat][2 * ((int64_t)t * tiles + i) + 1];
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      d += __shfl_xor_sync(FULL, d, off);
      p += __shfl_xor_sync(FULL, p, off);
    }
    if (lane == 0) A.qout[mat][t] = (p > 0.0) ? sqrt(d) / sqrt(p) : 0.0;
  }
}


}  // namespace

// Tile width: the narrowest tile of whole format blocks (16*S columns, S a power of two
// <= 8, S | n/16) that gives every thread at least 16 rows per pass, so the two barriers of
// a pass stay a small share of it. Resident rows: as many whole sweeps (512/S rows) as fit
// in shared memory next to the scale codes of all m rows and the reduction buffers. Depends
// on the shape, format and input type only (the Q-change trace shrinks R, which moves rows
// between shared memory and L2 but changes no result).
bool plan_solve(int64_t m, int64_t n, int kind, int group, int esize, bool qch, SolvePlan* p) {
  const int B = fmt_block(kind, group);
  if (B == 0 || m <= 0 || n <= 0 || n % B || m > (1 << 24)) return false;
  const int LPB = B / 16;
  const int scb = fmt_scale_bytes(kind);
  // Tile width: at least 16 rows per thread and pass (S doubles while fewer), and up to 32
  // while the rows that the resident CTAs stream from L2 every pass (all but the R in shared
  // memory, one CTA per SM) stay within a share of L2. More rows per pass spread the per-pass
  // column reduction and barriers over more work; a wider tile keeps fewer rows resident
  // (8B layer set: MXFP4 72.3 -> 69.4 ms per step, NVFP4 solve kernel -1.1%).
  auto streamed_bytes = [&](int s) -> int64_t {
    const SolveSmem b0 = solve_smem((int)m, 0, s, LPB, esize, scb, qch);
    const int ng = SOLVE_NT / s;
    const int64_t rb = (int64_t)16 * s * esize;
    if (b0.total + 128 > SOLVE_SMEM_MAX) return INT64_MAX;
    const int64_t r = (int64_t)(SOLVE_SMEM_MAX - b0.total - 128) / rb / ng * ng;
    return std::max<int64_t>(0, m - r) * rb * 148;
  };
  constexpr int64_t L2_STREAM_BUDGET = 48ll << 20;
  int S = LPB;
  while (S < 8 && n % (32 * S) == 0 &&
         (m * S < (int64_t)16 * SOLVE_NT ||
          (m * S < (int64_t)32 * SOLVE_NT &&
           streamed_bytes(2 * S) <= L2_STREAM_BUDGET)))
    S *= 2;
  const int NG = SOLVE_NT / S;
  const SolveSmem base = solve_smem((int)m, 0, S, LPB, esize, scb, qch);
  if (base.total + 128 > SOLVE_SMEM_MAX) return false;
  const int64_t row_bytes = (int64_t)16 * S * esize;
  int64_t R = (int64_t)(SOLVE_SMEM_MAX - base.total - 128) / row_bytes / NG * NG;
  R = std::min<int64_t>(R, (m + NG - 1) / NG * NG);
  const SolveSmem l = solve_smem((int)m, (int)R, S, LPB, esize, scb, qch);
  if (l.total > SOLVE_SMEM_MAX) return false;
  p->S = S;
  p->R = (int)R;
  p->tiles = (int)(n / (16 * S));
  p->smem = l.total;
  return true;
}

cudaError_t launch_solve(const SolveLaunch& L, int count, int kind, int group, int esize,
                         const SolvePlan& p, cudaStream_t s) {
  return launch_solve_formats<false>(L, count, kind, group, esize, p, s);
}

cudaError_t launch_solve_amax(const SolveLaunch& L, int count, int esize, cudaStream_t s) {
  // about 64 warps per SM over the whole launch, at most one warp per row
  const int warps = std::max(1, std::min(L.m, 148 * 64 / std::max(count, 1)));
  const int blocks = (warps + 7) / 8;
  if (esize == 4) solve_amax_kernel<4><<<dim3(blocks, count), 256, 0, s>>>(L);
  else solve_amax_kernel<2><<<dim3(blocks, count), 256, 0, s>>>(L);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_finalize(double* const* mse, double* const* ws_err, double* const* ws_wsq,
                            double* const* qchange, double* const* ws_qch, const int* tiles,
                            int count, int T, cudaStream_t s) {
  for (int base = 0; base < count; base += SOLVE_MAXMATS) {
    FinalizeArgs A = {};
    const int c = std::min(SOLVE_MAXMATS, count - base);
    for (int i = 0; i < c; ++i) {
      A.mse[i] = mse[base + i];
      A.err[i] = ws_err[base + i];
      A.wsq[i] = ws_wsq[base + i];
      A.qout[i] = qchange != nullptr ? qchange[base + i] : nullptr;
      A.qch[i] = ws_qch != nullptr ? ws_qch[base + i] : nullptr;
      A.tiles[i] = tiles[base + i];
    }
    A.T = T;
    const int warps = 8;
    finalize_kernel<<<dim3((T + 1 + warps - 1) / warps, c), warps * 32, 0, s>>>(A);
    count_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace dq
