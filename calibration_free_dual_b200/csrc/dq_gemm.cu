// dq_gemm.cu — the W4A4 GEMM that consumes the solver's and the activation quantizer's codes:
// y[t, i] = sum_j (d q_x)[t, j] (r q)[i, j] (NVFP4: E2M1 elements, E4M3 block scales per 16
// elements, one fp32 tensor scale per operand). The deployment side of DualQuant (ai4snews
// summary, paragraph 4: a real packed W4A4 inference path); the column scale c has already
// moved into the activation (dq_act_quant), so the GEMM sees two block-scaled operands.
//
// sm_100a design: 5th-generation tensor cores, block-scaled, warp-specialized. One CTA (six
// warps, two per SM) owns a 128 x 128 output tile accumulated in tensor memory (TMEM) by
// tcgen05.mma.kind::mxf4nvf4.block_scale (M = 128, N = 128, K = 64 per instruction):
//   * warp 0 (one lane) produces: per 256-wide K slice, bulk copies of the scale factors
//     (completing on the slice's "sf_full" mbarrier) and two TMA tile loads (128-byte
//     swizzle) of the packed E2M1 codes (on its "full" mbarrier); three slices in flight;
//   * warps 2-5 move each slice's scale factors from shared memory into TMEM (tcgen05.st,
//     one 32-lane sub-partition per warp) and signal the slice's "sf_ready" mbarrier, which
//     keeps those copies out of the tensor pipe (tcgen05.cp there serialises with the MMAs);
//   * warp 1 (one lane) issues the slice's four MMAs once "full" and "sf_ready" have
//     completed and commits them to the slice's "empty" mbarrier;
//   * after the last commit, warps 2-5 read the accumulator (tcgen05.ld), apply the two
//     tensor scales, stage the tile in the idle slice buffers as 32 x 32 blocks and write
//     them with TMA tensor stores (row stores when the output allows no tensor map).
// The scale factors are first re-laid (one small pre-pass launch for both operands) into the
// 128-row x 4 interleaving the tensor core reads, so a slice's scale factors are one
// contiguous copy.
// Every mbarrier wait is bounded by the global timer; on timeout the kernel raises the error
// word, frees its TMEM and returns.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <cuda.h>   // CUtensorMap and its enums (the encoder is fetched from the driver)

#include "dq_device.cuh"
#include "dq_internal.h"
#include "dq_gemm.h"

namespace dq {
namespace {

constexpr int GT = 192;                 // threads per CTA: producer, MMA, 4 scale/epilogue warps
constexpr unsigned FULL_MASK = 0xFFFFFFFFu;
// 128 x 128 tiles with three K slices in flight let two CTAs share an SM, so one CTA's set-up
// and epilogue overlap the other's MMAs: measured 10-20% faster than 128 x 256 tiles with
// four slices and one CTA per SM
constexpr int BM = 128, BN = 128;       // output tile (tokens x weight rows)
constexpr int BKE = 256;                // K elements per slice (NKB MMAs of K = 64)
constexpr int NKB = BKE / 64;
constexpr int BKB = BKE / 2;            // bytes of packed E2M1 per row per slice (128)
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BKB;       // 16 KB
constexpr int B_BYTES = BN * BKB;       // 16 KB
constexpr int SFA_BYTES = BM * BKE / 16;   // NKB blocks of 512 (one per MMA)
constexpr int SFB_BYTES = BN * BKE / 16;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;   // 36 KB
constexpr int BAR_OFF = STAGES * STAGE_BYTES;
constexpr int SMEM_NEED = BAR_OFF + 128 + 1024;    // barriers, TMEM slot, 1024-byte alignment
// with two CTAs per SM, more than a third of the SM's shared memory keeps a third CTA (and its
// TMEM allocation) off the SM
constexpr int SMEM_BYTES = SMEM_NEED;
constexpr uint32_t SF_COL0 = BN;                          // after the fp32 accumulator
constexpr uint32_t SF_COLS_PER_STAGE = 8 * NKB;           // SFA NKB MMAs x 4, SFB NKB x 4
constexpr uint32_t TMEM_COLS = 256;
constexpr int CTAS_PER_SM = 2;
constexpr int SMEM_LAUNCH = SMEM_BYTES < 80 * 1024 ? 80 * 1024 : SMEM_BYTES;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s: far beyond any slice's work

static_assert(NKB == 2 || NKB == 4, "slice of 2 or 4 MMAs");
static_assert(STAGE_BYTES % 1024 == 0, "1024-byte aligned slices (128-byte swizzle)");
static_assert(SMEM_LAUNCH * CTAS_PER_SM <= 226 * 1024, "shared memory");
static_assert(SF_COL0 + STAGES * SF_COLS_PER_STAGE <= TMEM_COLS, "TMEM columns");
static_assert(8 * (4 * STAGES + 1) + 8 <= 128, "barrier block");
static_assert(BM * BN * 4 <= STAGES * STAGE_BYTES, "epilogue staging fits in the slice buffers");

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- TMA tile loads and bulk copies, completing on an mbarrier (byte count)
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// shared -> global tile store through a tensor map (bulk-group completion)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
      :: "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(src) : "memory");
}

// ---- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes)
               : "memory");
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
// shared-memory matrix descriptor (sm_100 version 1): start address, leading and stride
// byte offsets, layout type (0: no swizzle, 2: 128-byte swizzle)
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}
// K-major operand slice written by a 128-byte-swizzled TMA box of 128-byte rows: 8-row
// groups 1024 bytes apart; an MMA's K = 64 slice starts 32 bytes further per step
__device__ __forceinline__ uint64_t operand_desc(uint32_t addr) { return smem_desc(addr, 16, 1024, 2); }
// 32 lanes x N consecutive 32-bit columns (N = 16 or 32) from registers into this warp's
// TMEM sub-partition
template <int N>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&r)[N]) {
  if constexpr (N == 32) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
           "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
           "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
           "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
           "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
  } else {
    static_assert(N == 16, "16 or 32 columns");
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16};"
        :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
           "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
           "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
  }
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
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


// instruction descriptor: A, B E2M1 (1), scale factors UE4M3 (0), K-major, M = BM, N = BN
constexpr uint32_t IDESC_NVFP4 = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                 ((uint32_t)(BM >> 4) << 24);

// Scale codes [rows, K/16] -> [row block of 128][K/64][512 bytes]: in each 512-byte block the
// four scales of row r of the block (for one MMA's 64 elements) sit at (r % 32) * 16 +
// (r / 32) * 4, so lane l of every TMEM sub-partition takes the 16 bytes at l * 16 and the
// tensor core picks the 4 bytes of its row group. Rows in [rows, rows_pad) are 0.
// One CTA re-lays SF_G groups of 4 scale bytes for one block of 128 rows of one operand
// (blockIdx.x: activation row blocks first, then weight row blocks; blockIdx.y: group chunk)
// through shared memory, with row-contiguous reads and block-contiguous writes.
constexpr int SF_G = 32;
__global__ void __launch_bounds__(256)
sf_interleave_kernel(const uint8_t* __restrict__ xs, int64_t T, int64_t tblk,
                     const uint8_t* __restrict__ ws, int64_t N, int64_t K,
                     uint8_t* __restrict__ sfa, uint8_t* __restrict__ sfb) {
  __shared__ uint32_t tile[SF_G][129];                 // [group][output word], padded
  const int64_t kq = K / 64;
  const bool act = (int64_t)blockIdx.x < tblk;
  const int64_t rb = act ? (int64_t)blockIdx.x : (int64_t)blockIdx.x - tblk;
  const uint8_t* src = act ? xs : ws;
  const int64_t rows = act ? T : N;
  uint8_t* dst = act ? sfa : sfb;
  const int64_t g0 = (int64_t)blockIdx.y * SF_G;
  const int ng = (int)((kq - g0) < SF_G ? (kq - g0) : SF_G);
  for (int i = threadIdx.x; i < 128 * SF_G; i += blockDim.x) {
    const int r = i / SF_G, gg = i % SF_G;
    const int64_t row = rb * 128 + r;
    uint32_t v = 0u;
    if (gg < ng && row < rows)
      v = *reinterpret_cast<const uint32_t*>(src + row * (K / 16) + 4 * (g0 + gg));
    tile[gg][(r & 31) * 4 + (r >> 5)] = v;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < ng * 128; i += blockDim.x) {
    const int gg = i / 128, w = i % 128;
    reinterpret_cast<uint32_t*>(dst + (rb * kq + g0 + gg) * 512)[w] = tile[gg][w];
  }
}

__global__ void __launch_bounds__(GT, CTAS_PER_SM)
w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmY, const __grid_constant__ GemmArgs A) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t t0 = (int64_t)blockIdx.y * BM, n0 = (int64_t)blockIdx.x * BN;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;               // 1024-byte aligned slices
  unsigned char* base_ptr = smem_raw + (sbase - raw);
  const uint32_t full0 = sbase + BAR_OFF;                      // full[s]    = full0 + 8s
  const uint32_t empty0 = full0 + 8 * STAGES;                  // empty[s]   = empty0 + 8s
  const uint32_t sfrdy0 = empty0 + 8 * STAGES;                 // sf_ready[s] = sfrdy0 + 8s
  const uint32_t sffull0 = sfrdy0 + 8 * STAGES;                // sf_full[s]  = sffull0 + 8s
  const uint32_t accbar = sffull0 + 8 * STAGES;                // accumulator complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + BAR_OFF + 8 * (4 * STAGES + 1));
  volatile int* fail = reinterpret_cast<volatile int*>(base_ptr + BAR_OFF + 8 * (4 * STAGES + 2));

  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
  if (tid == 32) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
      mbar_init(sfrdy0 + 8 * s, 4);
      mbar_init(sffull0 + 8 * s, 1);
    }
    mbar_init(accbar, 1);
    *fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nk = (int)((A.K + BKE - 1) / BKE);
  const int64_t kq = A.K / 64;

  if (warp == 0 && lane == 0) {
    // ---- producer
    for (int k = 0; k < nk; ++k) {
      const int s = k % STAGES;
      const uint32_t use = (uint32_t)(k / STAGES);             // how often slot s was used
      if (!mbar_wait(empty0 + 8 * s, (use & 1u) ^ 1u)) { *fail = 1; break; }
      if (*fail) break;
      const int nkb = (int)((kq - (int64_t)NKB * k) < NKB ? (kq - (int64_t)NKB * k) : NKB);
      const uint32_t sf_bytes = 512u * nkb;
      const uint32_t st = sbase + s * STAGE_BYTES;
      // the small scale-factor copies first, on their own barrier: their trip into TMEM
      // overlaps the operand tiles' arrival
      mbar_expect_tx(sffull0 + 8 * s, 2 * sf_bytes);
      bulk_load(st + A_BYTES + B_BYTES, A.sfa + ((t0 >> 7) * kq + (int64_t)NKB * k) * 512, sf_bytes,
                sffull0 + 8 * s);
      bulk_load(st + A_BYTES + B_BYTES + SFA_BYTES, A.sfb + ((n0 >> 7) * kq + (int64_t)NKB * k) * 512,
                sf_bytes, sffull0 + 8 * s);
      mbar_expect_tx(full0 + 8 * s, A_BYTES + B_BYTES);
      tma_load_2d(st, &tmA, k * BKB, (int)t0, full0 + 8 * s);
      tma_load_2d(st + A_BYTES, &tmB, k * BKB, (int)n0, full0 + 8 * s);
    }
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issue: the slice's operands (full) and its scale factors in TMEM (sf_ready)
    bool ok = true;
    for (int k = 0; k < nk; ++k) {
      const int s = k % STAGES;
      const uint32_t par = (uint32_t)(k / STAGES) & 1u;
      if (!mbar_wait(full0 + 8 * s, par) || !mbar_wait(sfrdy0 + 8 * s, par) || *fail) {
        *fail = 1;
        ok = false;
        break;
      }
      tc_fence_after();
      const int nkb = (int)((kq - (int64_t)NKB * k) < NKB ? (kq - (int64_t)NKB * k) : NKB);
      const uint32_t st = sbase + s * STAGE_BYTES;
      // SFA of MMA kb: TMEM columns +4kb; SFB: +4NKB +4kb
      const uint32_t tsf = tmem + SF_COL0 + SF_COLS_PER_STAGE * s;
      for (int kb = 0; kb < nkb; ++kb)
        mma_nvfp4(tmem, operand_desc(st + 32 * kb), operand_desc(st + A_BYTES + 32 * kb),
                  IDESC_NVFP4, (k > 0 || kb > 0) ? 1u : 0u, tsf + 4 * kb,
                  tsf + 4 * NKB + 4 * kb);
      mma_commit(empty0 + 8 * s);
    }
    if (ok) mma_commit(accbar);
  } else if (warp >= 2) {
    // TMEM sub-partition warp % 4: lanes (and accumulator rows) 32 * (warp % 4) ...
    const int sp = warp & 3;
    const uint32_t lane_base = tmem + ((uint32_t)(sp * 32) << 16);
    // ---- scale factors of every slice into TMEM. Each 512-byte block holds the scales of
    // one MMA for 128 rows, row r at (r % 32) * 16 + (r / 32) * 4: every sub-partition gets
    // the same 16 bytes per lane, and the tensor core picks the 4 bytes of its row group.
    bool ok = true;
    for (int k = 0; k < nk && ok; ++k) {
      const int s = k % STAGES;
      const uint32_t par = (uint32_t)(k / STAGES) & 1u;
      int got = 0;
      if (lane == 0) got = (mbar_wait(sffull0 + 8 * s, par) && !*fail) ? 1 : 0;
      ok = __shfl_sync(FULL_MASK, got, 0) != 0;
      if (!ok) break;
      const unsigned char* sfs = base_ptr + s * STAGE_BYTES + A_BYTES + B_BYTES + lane * 16;
      uint32_t r[8 * NKB];
#pragma unroll
      for (int kb = 0; kb < NKB; ++kb) {
        const uint4 a = *reinterpret_cast<const uint4*>(sfs + kb * 512);
        const uint4 b = *reinterpret_cast<const uint4*>(sfs + SFA_BYTES + kb * 512);
        r[4 * kb + 0] = a.x; r[4 * kb + 1] = a.y; r[4 * kb + 2] = a.z; r[4 * kb + 3] = a.w;
        r[4 * NKB + 4 * kb + 0] = b.x; r[4 * NKB + 4 * kb + 1] = b.y;
        r[4 * NKB + 4 * kb + 2] = b.z; r[4 * NKB + 4 * kb + 3] = b.w;
      }
      tmem_st<8 * NKB>(lane_base + SF_COL0 + SF_COLS_PER_STAGE * s, r);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sfrdy0 + 8 * s);
    }
    // ---- epilogue: accumulator -> scaled fp32 -> this warp's 32 rows, staged in the (now
    // idle) slice buffers as four 32 x 32 blocks of 128-byte rows, 16-byte chunks XOR-swizzled
    // by row (the 128-byte TMA swizzle: conflict-free writes of a row per lane) -> TMA tensor
    // stores of the four blocks (rows and columns past T, N clipped), or, when the output's
    // pitch or base does not allow a tensor map, row-contiguous stores by the warp
    if (ok) {
      int got = 0;
      if (lane == 0) got = (mbar_wait(accbar, 0) && !*fail) ? 1 : 0;
      ok = __shfl_sync(FULL_MASK, got, 0) != 0;
    }
    if (ok) {
      tc_fence_after();
      const float scale = __fmul_rn(*A.xst, *A.wst);
      unsigned char* stage = base_ptr + sp * (BN / 32) * 4096;   // 1024-byte aligned blocks
#pragma unroll 1
      for (int cb = 0; cb < BN / 32; ++cb) {
        float v[32];
        tmem_ld32(lane_base + cb * 32, v);
        float4* blk = reinterpret_cast<float4*>(stage + cb * 4096);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          blk[lane * 8 + (j ^ (lane & 7))] =
              make_float4(v[4 * j] * scale, v[4 * j + 1] * scale, v[4 * j + 2] * scale,
                          v[4 * j + 3] * scale);
      }
      if (A.store_tma) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          for (int cb = 0; cb < BN / 32; ++cb)
            if (n0 + cb * 32 < A.N && t0 + sp * 32 < A.T)        // boxes wholly outside: none
              tma_store_2d(&tmY, smem_u32(stage + cb * 4096), (int)(n0 + cb * 32),
                           (int)(t0 + sp * 32));
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
        __syncwarp();
      } else {
        __syncwarp();
        const int cb = lane >> 3, j = lane & 7;                   // this lane's 4 columns
        const int64_t c0 = n0 + cb * 32 + 4 * j;
        const int64_t ncols = A.N - c0;                           // columns left from c0
        const bool vec = ((A.ldy & 3) == 0) && ((reinterpret_cast<uintptr_t>(A.y) & 15u) == 0);
        const float4* blk = reinterpret_cast<const float4*>(stage + cb * 4096);
#pragma unroll 4
        for (int rr = 0; rr < 32; ++rr) {
          const int64_t t = t0 + sp * 32 + rr;
          if (t >= A.T) break;
          const float4 o = blk[rr * 8 + (j ^ (rr & 7))];
          float* dst = A.y + t * A.ldy + c0;
          if (ncols >= 4 && vec) {
            *reinterpret_cast<float4*>(dst) = o;
          } else {
            if (ncols > 0) dst[0] = o.x;
            if (ncols > 1) dst[1] = o.y;
            if (ncols > 2) dst[2] = o.z;
            if (ncols > 3) dst[3] = o.w;
          }
        }
      }
    } else if (lane == 0) {
      *fail = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *fail) atomicOr(A.err_word, ERRBIT_TIMEOUT);
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// cuTensorMapEncodeTiled from the driver (no link dependency on libcuda)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [rows, K/2] bytes, box of box_rows rows x 128 bytes, 128-byte swizzle, zero fill outside
bool make_codes_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t K,
                    uint32_t box_rows) {
  EncodeTiledFn fn = encoder();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  const cuuint32_t box[2] = {(cuuint32_t)BKB, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// y [rows, ldy] fp32, box of 32 rows x 32 floats (128 bytes), 128-byte swizzle; needs a
// 16-byte aligned base and a row pitch of a multiple of 16 bytes
bool make_out_map(CUtensorMap* map, float* y, int64_t rows, int64_t cols, int64_t ldy) {
  EncodeTiledFn fn = encoder();
  if (fn == nullptr || (reinterpret_cast<uintptr_t>(y) & 15u) != 0 || (ldy & 3) != 0) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ldy * 4)};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, y, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

}  // namespace

// W as [m][n/16][16] (rows, 16-column pieces, columns), box {16, S, solve_box_rows(S)}: a box
// is S pieces of solve_box_rows(S) rows, laid out row-major with the 32-byte (bf16) or 64-byte
// (fp32) swizzle, i.e. 16-byte chunk h of piece P at chunk 2P + (h ^ bit 2 of P), resp.
// 4P + (h ^ bits 1-2 of P): the order in which the solve kernel reads its resident rows.
// Rows past m read as zero.
bool make_w_map(CUtensorMap* map, const void* W, int64_t m, int64_t n, int64_t ldw, int esize,
                int S) {
  EncodeTiledFn fn = encoder();
  if (fn == nullptr || (esize != 2 && esize != 4) || n % 16 != 0) return false;
  const cuuint64_t dims[3] = {16, (cuuint64_t)(n / 16), (cuuint64_t)m};
  const cuuint64_t strides[2] = {(cuuint64_t)(16 * esize), (cuuint64_t)(ldw * esize)};
  const cuuint32_t box[3] = {16, (cuuint32_t)S, (cuuint32_t)solve_box_rows(S)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT32, 3,
            const_cast<void*>(W), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            esize == 2 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

size_t gemm_workspace_bytes(int64_t T, int64_t N, int64_t K, bool sfa_given) {
  // interleaved scale factors, rows padded to whole 128-row blocks
  return (size_t)((sfa_given ? 0 : round_up(T, BM)) + round_up(N, BN)) * (size_t)(K / 16) + 256;
}

cudaError_t launch_w4a4_gemm(const GemmArgs& A0, void* workspace, cudaStream_t s) {
  GemmArgs A = A0;
  const int64_t tpad = round_up(A.T, BM), npad = round_up(A.N, BN);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const bool sfa_given = A.sfa != nullptr;
  if (!sfa_given) A.sfa = ws;
  A.sfb = sfa_given ? ws : ws + tpad * (A.K / 16);
  // re-lay the scale factors (one launch; the weight's only when the activation's are given)
  const int64_t tblk = sfa_given ? 0 : tpad / BM;
  const dim3 sfgrid((unsigned)(tblk + npad / BN), (unsigned)((A.K / 64 + SF_G - 1) / SF_G), 1);
  sf_interleave_kernel<<<sfgrid, 256, 0, s>>>(A.xs, A.T, tblk, A.ws, A.N, A.K,
                                              const_cast<uint8_t*>(A.sfa),
                                              const_cast<uint8_t*>(A.sfb));
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  alignas(64) CUtensorMap ta, tb, ty;
  if (!make_codes_map(&ta, A.xq, A.T, A.K, BM) || !make_codes_map(&tb, A.wq, A.N, A.K, BN))
    return cudaErrorInvalidValue;
  A.store_tma = make_out_map(&ty, A.y, A.T, A.N, A.ldy) ? 1 : 0;
  if (!A.store_tma) memset(&ty, 0, sizeof(ty));          // not read by the kernel
  e = cudaFuncSetAttribute(w4a4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           SMEM_LAUNCH);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)(npad / BN), (unsigned)(tpad / BM), 1);
  timing_before(s);
  w4a4_gemm_kernel<<<grid, GT, SMEM_LAUNCH, s>>>(ta, tb, ty, A);
  e = cudaGetLastError();
  timing_after(s);
  count_launches(1);
  return e;
}

}  // namespace dq
