// dq_gemm.cu — the W4A4 GEMM that consumes the solver's and the activation quantizer's codes:
// y[t, i] = sum_j (d q_x)[t, j] (r q)[i, j] (NVFP4: E2M1 elements, E4M3 block scales per 16
// elements, one fp32 tensor scale per operand). The deployment side of DualQuant (ai4snews
// summary, paragraph 4: a real packed W4A4 inference path); the column scale c has already
// moved into the activation (dq_act_quant), so the GEMM sees two block-scaled operands.
//
// sm_100a design: 5th-generation tensor cores, block-scaled. One CTA (128 threads) owns a
// 128 x 128 output tile, accumulated in tensor memory (TMEM) by
// tcgen05.mma.kind::mxf4nvf4.block_scale (M = 128, N = 128, K = 64 per instruction), issued by
// one thread. The K loop is double-buffered: all threads stage the next 256-wide K slice of
// both operands into shared memory (cp.async, canonical K-major no-swizzle core-matrix layout)
// and its scale factors in the 128 x 4 interleaved layout the tensor core reads, while the
// tensor core works on the current slice; the scale factors go to TMEM with tcgen05.cp. The
// epilogue reads the accumulator with tcgen05.ld, multiplies by the two tensor scales and
// stores fp32. Every wait on an mbarrier is bounded: on timeout the kernel raises the error
// word, drains its own copies, frees its TMEM and returns.
#include <cstdint>

#include "dq_device.cuh"
#include "dq_internal.h"

namespace dq {
namespace {

constexpr int GT = 128;                 // threads per CTA
constexpr int BM = 128, BN = 128;       // output tile (tokens x weight rows)
constexpr int BKE = 256;                // K elements per stage (4 MMAs of K = 64)
constexpr int BKB = BKE / 2;            // bytes of packed E2M1 per row per stage
constexpr int STAGES = 2;
constexpr int OP_BYTES = BM * BKB;      // one operand's stage: 16 KB
constexpr int SF_BYTES = BM * BKE / 16; // one operand's scale factors per stage: 2 KB
constexpr int STAGE_BYTES = 2 * OP_BYTES + 2 * SF_BYTES;
constexpr int BAR_OFF = STAGES * STAGE_BYTES;
constexpr int SMEM_BYTES = 80 * 1024;   // > 1/3 of the SM: at most two CTAs (and 2 x 256 TMEM
                                        // columns) per SM, so a TMEM allocation never waits
constexpr uint32_t TMEM_COLS = 256;     // accumulator 128 + scale factors 2 x (16 + 16)
constexpr uint32_t SFA_COL = 128, SFB_COL = 160;   // + 16 per buffer
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s: far beyond any stage's work

static_assert(BAR_OFF + 64 <= SMEM_BYTES, "shared memory layout");

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- cp.async (16 bytes, L2 only; 4 bytes) with zero fill when src_size is 0
__device__ __forceinline__ void cp16(uint32_t dst, const void* src, uint32_t src_size) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src), "r"(src_size));
}
__device__ __forceinline__ void cp4(uint32_t dst, const void* src, uint32_t src_size) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" :: "r"(dst), "l"(src), "r"(src_size));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N)); }

// ---- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count));
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// bounded wait for the phase with the given parity to complete; false after WAIT_LIMIT_NS
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_try(bar, parity))
    if (global_ns() - t0 > WAIT_LIMIT_NS) return false;
  return true;
}

// ---- tensor memory and the tensor core (tcgen05)
__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               :: "r"(slot), "r"(ncols) : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
               :: "r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// shared-memory matrix descriptor: no swizzle, K-major canonical layout of 8-row x 16-byte
// core matrices; lbo = byte distance between the two 16-byte K halves an MMA reads, sbo =
// byte distance between consecutive groups of 8 rows; version 1 (sm_100)
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}
// 32 rows x 128 bits of scale factors from shared memory to TMEM, replicated into the four
// 32-lane sub-partitions
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(sdesc)
               : "memory");
}
// D (+)= A x B^T with E2M1 operands and E4M3 scale factors per 16 elements
__device__ __forceinline__ void mma_nvfp4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate, uint32_t tsfa,
                                          uint32_t tsfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      :: "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(bar) : "memory");
}
// 32 lanes x 32 consecutive fp32 columns (each thread: its lane, 32 values)
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// instruction descriptor: A, B E2M1 (1), scale factors UE4M3 (0), K-major, M = 128, N = 128
constexpr uint32_t IDESC_NVFP4 = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                 ((uint32_t)(BM >> 4) << 24);

// One stage of loads: the 256-wide K slice [k0, k0 + 256) of the 128 rows [row0, row0 + 128)
// of one operand (codes [rows, K/2] bytes, scale codes [rows, K/16] bytes).
//   codes -> smem offset kc*2048 + (row/8)*128 + (row%8)*16 for the 16-byte chunk kc (32
//            elements): MMA kb reads chunks 2kb, 2kb+1 (lbo 2048, sbo 128);
//   scale codes -> the 512-byte block of MMA kb, byte (row%32)*16 + (row/32)*4 + s for its
//            s-th scale (s < 4): the 128 x 4 interleaving tcgen05.cp 32x128b.warpx4 expects.
// Rows past `rows` and columns past K are zero-filled (scale 0 = no contribution).
__device__ __forceinline__ void load_stage(const uint8_t* codes, const uint8_t* scales,
                                           int64_t rows, int64_t K, int64_t row0, int64_t k0,
                                           uint32_t s_codes, uint32_t s_sf, int tid) {
  const int64_t kbytes = K / 2, kscales = K / 16;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = tid + GT * i;                    // 1024 chunks: 8 rows x 8 chunks x 16 groups
    const int r8 = c & 7, kc = (c >> 3) & 7, rg = c >> 6;
    const int row = rg * 8 + r8;
    const int64_t grow = row0 + row;
    const bool ok = grow < rows && k0 + 32 * kc < K;
    const uint8_t* src = ok ? codes + grow * kbytes + k0 / 2 + 16 * kc : codes;
    cp16(s_codes + kc * 2048 + rg * 128 + r8 * 16, src, ok ? 16u : 0u);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = tid + GT * i;                    // 512 groups of 4 scales: 128 rows x 4 MMAs
    const int row = c & 127, kb = c >> 7;
    const int64_t grow = row0 + row;
    const bool ok = grow < rows && k0 + 64 * kb < K;
    const uint8_t* src = ok ? scales + grow * kscales + k0 / 16 + 4 * kb : scales;
    cp4(s_sf + kb * 512 + (row & 31) * 16 + (row >> 5) * 4, src, ok ? 4u : 0u);
  }
}

__global__ void __launch_bounds__(GT, 1) w4a4_gemm_kernel(const __grid_constant__ GemmArgs A) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t t0 = (int64_t)blockIdx.y * BM, n0 = (int64_t)blockIdx.x * BN;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + BAR_OFF;           // mbar[0], mbar[1]: MMAs of a stage done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + BAR_OFF + 16);

  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
  if (tid == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar0 + 8, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int nk = (int)((A.K + BKE - 1) / BKE);
  uint32_t phase[STAGES] = {0u, 0u};
  bool timeout = false;

  auto stage_addr = [&](int buf) { return sbase + buf * STAGE_BYTES; };
  auto issue = [&](int k, int buf) {
    const uint32_t s = stage_addr(buf);
    load_stage(A.xq, A.xs, A.T, A.K, t0, (int64_t)k * BKE, s, s + 2 * OP_BYTES, tid);
    load_stage(A.wq, A.ws, A.N, A.K, n0, (int64_t)k * BKE, s + OP_BYTES,
               s + 2 * OP_BYTES + SF_BYTES, tid);
    cp_commit();
  };

  issue(0, 0);
  for (int k = 0; k < nk && !timeout; ++k) {
    const int buf = k & 1;
    if (k + 1 < nk) {
      if (k >= 1) {
        // the MMAs of stage k-1 read buffer (k+1)&1: thread 0 waits for them (bounded), the
        // barrier makes the outcome uniform before anyone refills the buffer
        const int pb = (k + 1) & 1;
        const bool ok = tid != 0 || mbar_wait(bar0 + 8 * pb, phase[pb]);
        phase[pb] ^= 1u;
        timeout = __syncthreads_or(!ok) != 0;
      }
      if (timeout) break;
      issue(k + 1, (k + 1) & 1);
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    fence_async_smem();              // this thread's copies, visible to the tensor core
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t s = stage_addr(buf);
      const int64_t left = (A.K - (int64_t)k * BKE + 63) / 64;
      const int nkb = left < 4 ? (int)left : 4;
      const uint32_t tsfa = tmem + SFA_COL + 16 * buf, tsfb = tmem + SFB_COL + 16 * buf;
      for (int kb = 0; kb < nkb; ++kb) {
        tmem_cp_sf(tsfa + 4 * kb, smem_desc(s + 2 * OP_BYTES + kb * 512, 0, 128));
        tmem_cp_sf(tsfb + 4 * kb, smem_desc(s + 2 * OP_BYTES + SF_BYTES + kb * 512, 0, 128));
      }
      for (int kb = 0; kb < nkb; ++kb) {
        const uint64_t ad = smem_desc(s + 2 * kb * 2048, 2048, 128);
        const uint64_t bd = smem_desc(s + OP_BYTES + 2 * kb * 2048, 2048, 128);
        mma_nvfp4(tmem, ad, bd, IDESC_NVFP4, (k > 0 || kb > 0) ? 1u : 0u, tsfa + 4 * kb,
                  tsfb + 4 * kb);
      }
      mma_commit(bar0 + 8 * buf);
    }
  }

  // the last stage's MMAs (in issue order after every earlier one); the outcome is made
  // uniform across the CTA before the epilogue's warp-collective TMEM loads
  if (!timeout && nk > 0) {
    const int lb = (nk - 1) & 1;
    const bool ok = tid != 0 || mbar_wait(bar0 + 8 * lb, phase[lb]);
    timeout = __syncthreads_or(!ok) != 0;
  }
  cp_wait<0>();                      // no copy of ours is still in flight
  if (timeout) {
    if (tid == 0) atomicOr(A.err_word, ERRBIT_TIMEOUT);
  } else {
    tc_fence_after();
    const float scale = __fmul_rn(*A.xst, *A.wst);
    const int64_t t = t0 + warp * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll
    for (int cb = 0; cb < BN / 32; ++cb) {
      float v[32];
      tmem_ld32(lane_addr + cb * 32, v);
      if (t < A.T) {
        float* yrow = A.y + t * A.ldy + n0 + cb * 32;
        const int64_t rem = A.N - n0 - cb * 32;
        const int64_t ncols = rem < 32 ? rem : 32;
        if (ncols == 32 && (reinterpret_cast<uintptr_t>(yrow) & 15u) == 0) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(yrow + i) =
                make_float4(v[i] * scale, v[i + 1] * scale, v[i + 2] * scale, v[i + 3] * scale);
        } else {
          for (int i = 0; i < ncols; ++i) yrow[i] = v[i] * scale;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

size_t gemm_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_w4a4_gemm(const GemmArgs& A, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(w4a4_gemm_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((A.N + BN - 1) / BN), (unsigned)((A.T + BM - 1) / BM), 1);
  timing_before(s);
  w4a4_gemm_kernel<<<grid, GT, SMEM_BYTES, s>>>(A);
  e = cudaGetLastError();
  timing_after(s);
  count_launches(1);
  return e;
}

}  // namespace dq
