// dq_solve_kernel.cuh — the dual-scale BCD solve kernel (sm_100a), one column strip per CTA.
//
// Method: DualQuant ("DualQuant: Dual-scale Calibration-free Weight-and-Activation
// Quantization for LLMs", Abstract): W ~ diag(r) Q diag(c) fitted by block coordinate
// descent, every block updated in closed form; the quantizer is a black box and the scales
// are projected onto the format's admissible set after each update (acceptodds.com
// abstract of the same paper); the normalised-MSE trace of Figure 2 (b).
//
// B200 design. With r per (row, B-column block) and c per column, every step couples only
// columns of one block (r-step) or rows of one column (c-step), so the solve splits exactly
// into independent column strips. One CTA (512 threads, one per SM) owns a tile of
// TN = 16*S columns and ALL m rows of it, so every reduction of the solve is CTA-local and
// needs only __syncthreads:
//   * the first R rows of the tile stay in shared memory for the whole solve (copied once
//     from HBM by the tensor memory accelerator: tensor-map boxes whose swizzle is the row
//     loop's bank-conflict-free order); the remaining rows are read again from L2 on every
//     pass with 256-bit loads marked evict-last (the streamed rows of all resident CTAs stay
//     far below the 126 MB L2), the next row in flight while the current one is processed;
//   * each thread owns one 16-column piece of a set of rows; LPB = B/16 neighbouring lanes
//     share one format block and combine its r-step sums with xor shuffles;
//   * Q-, r- and c-step run per row in registers with packed fp32x2 arithmetic
//     (FMUL2/FFMA2) and the E2M1/E4M3 cvt instructions;
//   * per pass, the per-column sums N_j, D_j go through a butterfly inside each warp (fp32)
//     and a fixed binary64 tree across the 16 warps; the warps that own the tree also form
//     the closed-form c_j and the pass's error terms. Two barriers per pass, no spin-waits;
//   * iterations 0 and 1 share the first pass (iteration 1's codes are iteration 0's), so
//     T iterations take T passes over the tile.
#pragma once

#include <algorithm>
#include <type_traits>

#include "dq_device.cuh"
#include "dq_internal.h"

namespace dq {
namespace {

constexpr unsigned FULL = 0xFFFFFFFFu;
constexpr int NWARP = SOLVE_NT / 32;

// ---- the resident-row copy by the tensor memory accelerator: boxes of the W tensor map
// land in shared memory and complete on one mbarrier (transaction bytes)
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void tma_box_3d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                           int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];"
      :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
// bounded wait for phase 0 of the copy's mbarrier: false after 2 s of global time
__device__ __forceinline__ bool copy_wait(uint32_t bar) {
  uint64_t t0, t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (;;) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar) : "memory");
    if (ok) return true;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 > 2000000000ull) return false;
  }
}

// 16-byte chunk position of chunk h of piece P (the 16 columns one thread owns in one row;
// row-major [R][TN] tile, CPP chunks per piece). The 8 lanes of a quarter warp read 8
// consecutive pieces; the swizzle spreads them over the 8 bank groups.
template <int CPP>
__device__ __forceinline__ int chunk_pos(int P, int h) {
  if constexpr (CPP == 2) return 2 * P + (h ^ ((P >> 2) & 1));
  else return 4 * P + (h ^ ((P >> 1) & 3));
}

// One row piece as raw words (bf16: 8 words; fp32: 16 words).
template <int ESZ>
struct Raw {
  uint32_t u[ESZ * 4];
};

template <int ESZ>
__device__ __forceinline__ void unpack(const Raw<ESZ>& r, float2 (&w)[8]) {
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    if constexpr (ESZ == 2) w[p] = bf16x2_to_f2(r.u[p]);
    else w[p] = make_float2(__uint_as_float(r.u[2 * p]), __uint_as_float(r.u[2 * p + 1]));
  }
}

template <int ESZ>
__device__ __forceinline__ void zero(Raw<ESZ>& r) {
#pragma unroll
  for (int i = 0; i < ESZ * 4; ++i) r.u[i] = 0u;
}

// 32 bytes from L2, not allocated in L1, kept in L2 ahead of normal lines (evict-last):
// these rows are read again on every pass.
__device__ __forceinline__ void ldg256_keep(const void* p, uint32_t* d) {
  asm volatile(
      "ld.global.nc.L1::no_allocate.L2::evict_last.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]), "=r"(d[6]),
        "=r"(d[7])
      : "l"(p));
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// A streamed row piece: 256-bit loads when every row start is 32-byte aligned, else 128-bit.
template <int ESZ>
__device__ __forceinline__ void load_global(const char* p, bool wide, Raw<ESZ>& r) {
  if (wide) {
#pragma unroll
    for (int h = 0; h < ESZ / 2; ++h) ldg256_keep(p + 32 * h, r.u + 8 * h);
  } else {
#pragma unroll
    for (int h = 0; h < ESZ; ++h) {
      const uint4 v = ldg_stream(p + 16 * h);
      r.u[4 * h + 0] = v.x;
      r.u[4 * h + 1] = v.y;
      r.u[4 * h + 2] = v.z;
      r.u[4 * h + 3] = v.w;
    }
  }
}

// Butterfly reduction of 32 values over the 32/S lanes sharing piece s = lane % S.
// Lane L ends with the S totals of indices [L - s, L - s + S) (fixed order).
template <int S>
__device__ __forceinline__ void transpose_reduce(float (&v)[32], int lane) {
  int cnt = 32;
#pragma unroll
  for (int off = 16; off >= S; off >>= 1) {
    const int half = cnt >> 1;
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i < half) {
        const float send = upper ? v[i] : v[i + half];
        const float keep = upper ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(FULL, send, off);
      }
    }
    cnt = half;
  }
}

// One CTA: all m rows of the column tile [tile*TN, tile*TN + TN) of matrix blockIdx.y.
// EXT (the extended instantiation; the plain one updates both scales and records no Q-change):
// runtime flags select which scales the iterations update, and on request the Q-change
// trace of Figure 2 (a): from the second iteration on, every row re-quantizes W with the
// previous iteration's (r, c), kept in shared memory, and adds sum (q - q_prev)^2 and
// sum q_prev^2 (exact: multiples of 1/4 far below 2^24).
template <int ELEM, int SCALE, int LPB, int S, bool F32IN, bool EXT>
__global__ void __launch_bounds__(SOLVE_NT, 1)
solve_kernel(const __grid_constant__ SolveLaunch L) {
  constexpr int NT = SOLVE_NT, TN = 16 * S, NBLK = S / LPB, B = 16 * LPB;
  constexpr int NG = NT / S;             // rows covered by one sweep of all threads
  constexpr int ESZ = F32IN ? 4 : 2;
  constexpr int SCB = (SCALE == SCALE_BF16) ? 2 : 1;
  constexpr float QMAX = elem_qmax<ELEM>();
  constexpr bool BYTE_CODES = (ELEM == ELEM_INT8);        // one code byte per element
  static_assert(NBLK * LPB == S && S >= 1 && S <= 8, "tile shape");
  // code-shape choices by format (measured on the 8B layer set; results do not depend on
  // them): the three row loops pay for E4M3 (one-lane blocks) and the bf16-scale formats,
  // whose extra registers cost the E8M0 formats more than the per-row test saves
  constexpr bool SPLIT_ROWS = (SCALE != SCALE_E8M0);

  const int m = L.m, n = L.n, T = L.T, tiles = L.tiles;
  const int tile = blockIdx.x;
  const SolveMat& M = L.mats[blockIdx.y];
  const int col0 = tile * TN;
  const int nb = n / B;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = tid % S, g = tid / S, bl = s / LPB, lib = s % LPB;
  const bool wide = L.wide != 0;
  const char* gW = reinterpret_cast<const char*>(M.W) + (int64_t)(col0 + s * 16) * ESZ;
  const int64_t pitch = M.ldw * ESZ;

  extern __shared__ __align__(128) unsigned char smem[];
  const bool upd_r = !EXT || L.upd_r != 0, upd_c = !EXT || L.upd_c != 0;
  const bool qch = EXT && L.qch != 0;
  const SolveSmem lay = solve_smem(m, L.R, S, LPB, ESZ, SCB, qch);
  unsigned char* Wsm = smem + lay.w;
  void* codes_v = smem + lay.codes;
  float2* tbl = reinterpret_cast<float2*>(smem + lay.tbl);
  float* cvec = reinterpret_cast<float*>(smem + lay.cvec);
  float* icvec = reinterpret_cast<float*>(smem + lay.icvec);
  float* red = reinterpret_cast<float*>(smem + lay.red);
  double* errw = reinterpret_cast<double*>(smem + lay.cols);   // [S] per-warp error sums
  double* e0w = errw + 8;                                      // [NWARP] iteration-0 errors
  double* wsqw = e0w + NWARP;                                  // [NWARP] ||W||^2 sums
  void* pcodes_v = smem + lay.pcodes;                          // Q-change: previous codes
  float* picvec = reinterpret_cast<float*>(smem + lay.picvec); // Q-change: previous 1/c
  double* qred = reinterpret_cast<double*>(smem + lay.qred);   // Q-change: per-warp sums

  // Sweep k gives this thread row g + k*NG; with NG*S = NT its piece is number tid + NT*k of
  // the row-major tile and its block's scale code is number tid/LPB + k*NT/LPB.
  const int code0 = tid / LPB;
  auto code_at = [&](int k) -> uint32_t {
    if constexpr (SCB == 2) return reinterpret_cast<uint16_t*>(codes_v)[code0 + k * (NT / LPB)];
    else return reinterpret_cast<uint8_t*>(codes_v)[code0 + k * (NT / LPB)];
  };
  auto set_code = [&](int k, uint32_t code) {
    if constexpr (SCB == 2)
      reinterpret_cast<uint16_t*>(codes_v)[code0 + k * (NT / LPB)] = (uint16_t)code;
    else reinterpret_cast<uint8_t*>(codes_v)[code0 + k * (NT / LPB)] = (uint8_t)code;
  };
  auto pcode_at = [&](int k) -> uint32_t {
    if constexpr (SCB == 2) return reinterpret_cast<uint16_t*>(pcodes_v)[code0 + k * (NT / LPB)];
    else return reinterpret_cast<uint8_t*>(pcodes_v)[code0 + k * (NT / LPB)];
  };
  auto set_pcode = [&](int k, uint32_t code) {
    if constexpr (SCB == 2)
      reinterpret_cast<uint16_t*>(pcodes_v)[code0 + k * (NT / LPB)] = (uint16_t)code;
    else reinterpret_cast<uint8_t*>(pcodes_v)[code0 + k * (NT / LPB)] = (uint8_t)code;
  };

  // ---- rows [0, R) into shared memory (their only read from HBM), all in flight at once;
  // rows past m (only in the last sweep) are zero-filled and add nothing to any sum. With a
  // tensor map of W, one thread issues boxes of {16 columns, S pieces, BR rows} through the
  // tensor memory accelerator: the map's 32-byte (bf16) / 64-byte (fp32) swizzle puts every
  // 16-byte chunk where chunk_pos places it (the swizzle works on address bits, so the copy
  // needs the buffer aligned to the swizzle's 256- / 512-byte period). Otherwise every thread
  // issues asynchronous 16-byte copies. Awaited before the first pass; the iteration-0 pass
  // checks every row for non-finite values.
  const uint32_t wsm_addr = smem_addr(Wsm);
  const uint32_t wbar = smem_addr(smem + lay.bar);
  const bool tma = L.tma != 0 && L.R > 0 && (wsm_addr & (ESZ == 2 ? 255u : 511u)) == 0;
  if (tma) {
    // boxes that start below m (a box that runs past m is zero-filled beyond it); the rows of
    // boxes wholly past m (a 512-row sweep takes two boxes when S = 1) are zeroed here
    constexpr int BR = solve_box_rows(S);
    const int rtma = min(L.R, (m + BR - 1) / BR * BR);
    if (tid == 0) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" :: "r"(wbar) : "memory");
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                   :: "r"(wbar), "r"((uint32_t)rtma * TN * ESZ) : "memory");
      for (int r0 = 0; r0 < rtma; r0 += BR)
        tma_box_3d(wsm_addr + (uint32_t)r0 * TN * ESZ, &L.wmap[blockIdx.y], 0, tile * S, r0,
                   wbar);
    }
    uint4* zw = reinterpret_cast<uint4*>(Wsm + (size_t)rtma * TN * ESZ);
    for (int i = tid; i < (L.R - rtma) * TN * ESZ / 16; i += NT) zw[i] = make_uint4(0u, 0u, 0u, 0u);
  } else {
    constexpr int CH = TN * ESZ / 16;      // 16-byte chunks per row
    const char* base = reinterpret_cast<const char*>(M.W) + (int64_t)col0 * ESZ;
#pragma unroll 4
    for (int ch = tid; ch < L.R * CH; ch += NT) {
      const int row = ch / CH, part = ch % CH;
      const bool in = row < m;
      const char* src = base + (int64_t)(in ? row : 0) * pitch + part * 16;
      const uint32_t dst = wsm_addr + 16u * chunk_pos<ESZ>(row * S + part / ESZ, part % ESZ);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                   :: "r"(dst), "l"(src), "r"(in ? 16 : 0) : "memory");
    }
  }

  // ---- tensor scale (NVFP4) and the code -> (r, 1/r) table; bf16 scales: the table of
  // mantissa reciprocals
  float s_t = 1.0f;
  const float* rtab = reinterpret_cast<const float*>(tbl);
  if constexpr (SCALE == SCALE_BF16) {
    if (tid < 128) reinterpret_cast<float*>(tbl)[tid] = __frcp_rn(1.0f + (float)tid * 0.0078125f);
  }
  if constexpr (SCALE == SCALE_E4M3) {
    s_t = nvfp4_tensor_scale(__uint_as_float(*M.amax_bits));
    if (tid < 128) {
      const uint32_t code = (tid == 0 || tid == 127) ? 1u : (uint32_t)tid;
      const float r = __fmul_rn(s_t, e4m3_decode(code));
      tbl[tid] = make_float2(r, __frcp_rn(r));
    }
    if (tile == 0 && tid == 0 && M.tensor_scale != nullptr) *M.tensor_scale = s_t;
  }

  // ---- column scales: c0 or 1
  if (tid < TN) {
    float cj = 1.0f;
    if (M.c0 != nullptr) {
      cj = M.c0[col0 + tid];
      if (!(cj > 0.0f && cj <= 3.0e38f)) {
        atomicOr(L.err_word, ERRBIT_BADWARM);
        cj = 1.0f;
      }
    }
    cvec[tid] = cj;
    icvec[tid] = __frcp_rn(cj);
  }

  if (tma) {
    // (the barrier's initialisation is visible to all threads after this sync)
    __syncthreads();
    const bool ok = copy_wait(wbar);
    if (__syncthreads_or(!ok)) {
      if (tid == 0) atomicOr(L.err_word, ERRBIT_TIMEOUT);
      return;
    }
  } else {
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
  }

  float2 cc[8], ic[8];
  auto load_c = [&]() {
    const float4* cv = reinterpret_cast<const float4*>(cvec + s * 16);
    const float4* iv = reinterpret_cast<const float4*>(icvec + s * 16);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float4 a = cv[h], b = iv[h];
      cc[2 * h] = make_float2(a.x, a.y);
      cc[2 * h + 1] = make_float2(a.z, a.w);
      ic[2 * h] = make_float2(b.x, b.y);
      ic[2 * h + 1] = make_float2(b.z, b.w);
    }
  };
  load_c();

  const int RPT = (m + NG - 1) / NG;       // sweeps per pass (uniform: shuffles below)
  const int KS = min(L.R / NG, RPT);       // sweeps served from shared memory
  const int64_t qpitch = BYTE_CODES ? n : (n >> 1);         // code bytes per row

  // row piece of sweep k: shared memory (chunk h of piece tid + NT*k sits at
  // ESZ*(tid + NT*k) + (h ^ sw)), else L2, or zeros past the last row
  const uint4* smp = reinterpret_cast<const uint4*>(Wsm) + ESZ * tid;
  const int sw = (ESZ == 2) ? ((tid >> 2) & 1) : ((tid >> 1) & 3);
  const char* gp = gW + (int64_t)g * pitch;
  const int64_t gstep = (int64_t)NG * pitch;
  auto fetch = [&](int k, Raw<ESZ>& dst) {
    if (k < KS) {
#pragma unroll
      for (int h = 0; h < ESZ; ++h) {
        const uint4 v = smp[ESZ * NT * k + (h ^ sw)];
        dst.u[4 * h + 0] = v.x;
        dst.u[4 * h + 1] = v.y;
        dst.u[4 * h + 2] = v.z;
        dst.u[4 * h + 3] = v.w;
      }
    } else if (g + k * NG < m) {
      load_global<ESZ>(gp + k * gstep, wide, dst);
    } else {
      zero<ESZ>(dst);
    }
  };

  // per-column totals of the 32-value vectors (a: 16 columns, b: 16 columns) of all
  // threads; thread tid < 32*S (lane e of warp sj) returns the total of value e of piece sj
  auto column_totals = [&](const float2 (&a)[8], const float2 (&b)[8]) -> double {
    float v[32];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      v[2 * p] = a[p].x;
      v[2 * p + 1] = a[p].y;
      v[16 + 2 * p] = b[p].x;
      v[16 + 2 * p + 1] = b[p].y;
    }
    transpose_reduce<S>(v, lane);
#pragma unroll
    for (int i = 0; i < S; ++i) red[(warp * S + s) * 32 + (lane - s) + i] = v[i];
    __syncthreads();
    double tot = 0.0;
    if (tid < 32 * S) {
      double va[NWARP];
#pragma unroll
      for (int wp = 0; wp < NWARP; ++wp) va[wp] = (double)red[wp * S * 32 + tid];
#pragma unroll
      for (int st = 1; st < NWARP; st <<= 1) {
#pragma unroll
        for (int i = 0; i + st < NWARP; i += 2 * st) va[i] += va[i + st];
      }
      tot = va[0];
    }
    return tot;
  };

  double wsq_tile = 0.0;    // ||W||^2 of the tile (thread 0)

  // code -> scale: bf16 scales with the reciprocal table, the others as before
  auto dec = [&](uint32_t code) -> ScaleVal {
    if constexpr (SCALE == SCALE_BF16) return bf16_scale_decode_tab(code, rtab);
    else return scale_decode<SCALE>(code, tbl);
  };

  // One pass over all rows of the tile. INIT: iteration 0 (scales from absmax or r0,
  // c = c0); otherwise one BCD iteration (Q-step, r-step + projection, c-step). EMIT: the
  // returned state is written.
  //
  // FUSE (with INIT): iteration 0 and iteration 1 in one sweep. Iteration 1's Q-step sees the
  // state of iteration 0, so its codes are iteration 0's: the pass quantizes once, adds the
  // iteration-0 error sum (W - r q c)^2 directly, then runs iteration 1's r-step and c-step.
  auto pass = [&](auto init_tag, auto emit_tag, auto fuse_tag, const int t) {
    constexpr bool INIT = decltype(init_tag)::value;
    constexpr bool EMIT = decltype(emit_tag)::value;
    constexpr bool FUSE = INIT && decltype(fuse_tag)::value;
    constexpr bool ITER = !INIT || FUSE;     // the pass runs an iteration's r- and c-steps
    float2 accN[8], accD[8];
    float2 accW2 = make_float2(0.f, 0.f), accE0 = make_float2(0.f, 0.f);   // INIT, FUSE
    float2 accQd = make_float2(0.f, 0.f), accQp = make_float2(0.f, 0.f);   // Q-change
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      accN[p] = make_float2(0.f, 0.f);
      accD[p] = make_float2(0.f, 0.f);
    }
    bool bad = false;

    // the next row's piece and (after iteration 0) its scale are fetched one row ahead
    Raw<ESZ> buf;
    fetch(0, buf);
    ScaleVal scn;
    if constexpr (!INIT) scn = dec(code_at(0));
    // one row step; NEXT: which source the next row comes from (0: none, this is the last
    // row; 1: shared memory; 2: L2, or zeros past the last row; 3: tested per row; 4: L2, a
    // sweep with every row below m, 256-bit loads). With SPLIT_ROWS the source is fixed per
    // loop below, so the row steps carry no per-row test
    auto step = [&](const int k, auto next_tag) {
      constexpr int NEXT = decltype(next_tag)::value;
      [[maybe_unused]] const int row = g + k * NG;
      float2 w[8];
      unpack<ESZ>(buf, w);
      ScaleVal sc;
      uint32_t old_code = 0u;                 // the Q-change trace's previous scale code
      if constexpr (!INIT) {
        sc = scn;
        old_code = sc.code;
      }
      if constexpr (NEXT == 1) {
#pragma unroll
        for (int h = 0; h < ESZ; ++h) {
          const uint4 v = smp[ESZ * NT * (k + 1) + (h ^ sw)];
          buf.u[4 * h + 0] = v.x;
          buf.u[4 * h + 1] = v.y;
          buf.u[4 * h + 2] = v.z;
          buf.u[4 * h + 3] = v.w;
        }
      } else if constexpr (NEXT == 2) {
        if (g + (k + 1) * NG < m) load_global<ESZ>(gp + (k + 1) * gstep, wide, buf);
        else zero<ESZ>(buf);
      } else if constexpr (NEXT == 4) {
#pragma unroll
        for (int h = 0; h < ESZ / 2; ++h) ldg256_keep(gp + (k + 1) * gstep + 32 * h, buf.u + 8 * h);
      }
      if constexpr (NEXT == 3) {
        if (k + 1 < RPT) {
          fetch(k + 1, buf);
          if constexpr (!INIT) scn = dec(code_at(k + 1));
        }
      } else if constexpr (!INIT && NEXT != 0) {
        scn = dec(code_at(k + 1));
      }
      if constexpr (INIT) {
        // NaN-propagating maximum: a is non-finite exactly when one of the piece's values is
        float a = 0.0f;
#pragma unroll
        for (int p = 0; p < 8; ++p) a = max_nan(a, max_nan(fabsf(w[p].x), fabsf(w[p].y)));
        bad |= !isfinite(a);
#pragma unroll
        for (int off = 1; off < LPB; off <<= 1) a = fmaxf(a, __shfl_xor_sync(FULL, a, off));
        float v;
        if (M.r0 != nullptr) {
          v = (row < m) ? M.r0[(int64_t)row * nb + col0 / B + bl] : 1.0f;
        } else {
          v = (a > 0.0f) ? div_qmax<(int)QMAX>(a) : 1.0f;
        }
        sc = dec(project_code<SCALE>(v, s_t));
        old_code = sc.code;
      }

      // Q-step on the binary32 quotient fl32(fl32(w * 1/c) * 1/r)
      float2 q[8];
      [[maybe_unused]] uint32_t codes[4] = {0u, 0u, 0u, 0u};
      const float2 irr = make_float2(sc.ir, sc.ir);
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const float2 x = mul2(mul2(w[p], ic[p]), irr);
        if constexpr (EMIT && BYTE_CODES) codes[p >> 1] |= quant2<ELEM>(x, q[p]) << (16 * (p & 1));
        else if constexpr (EMIT) codes[p >> 2] |= quant2<ELEM>(x, q[p]) << (8 * (p & 3));
        else q[p] = quant2_value<ELEM>(x);
      }
      if constexpr (FUSE) {
        // iteration 0's error W - r q c, straight from its state (c: the initial column scales)
        const float2 nr = make_float2(-sc.r, -sc.r);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const float2 e = fma2(mul2(q[p], nr), cc[p], w[p]);
          accE0 = fma2(e, e, accE0);
        }
      }
      if constexpr (EXT && !INIT) {
        if (qch && t >= 2) {
          // q of the previous iteration, from its (r, c)
          const ScaleVal sp = dec(pcode_at(k));
          const float2 irp = make_float2(sp.ir, sp.ir);
          const float4* pv = reinterpret_cast<const float4*>(picvec + s * 16);
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float4 a = pv[h];
            const float2 pic[2] = {make_float2(a.x, a.y), make_float2(a.z, a.w)};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int pp = 2 * h + e;
              const float2 qp = quant2_value<ELEM>(mul2(mul2(w[pp], pic[e]), irp));
              const float2 d = fma2(qp, make_float2(-1.0f, -1.0f), q[pp]);
              accQd = fma2(d, d, accQd);
              accQp = fma2(qp, qp, accQp);
            }
          }
        }
      }

      if (ITER && upd_r) {
        // r-step: least squares over the block, then projection
        if constexpr (SCALE == SCALE_BF16) {
          // The fine bf16 scale grid: the block sums in binary32 first. Every term is >= 0
          // (a code has the sign of its weight), so the binary32 sums carry a relative error
          // of at most 13 and 14 units of binary32 rounding (the longest chain of roundings:
          // the product q c, 8 accumulations, the pair, 3 shuffle levels), and the correctly
          // rounded quotient v at most 28, i.e. under 28 ulps of v. bf16 rounds at the
          // binary32 patterns whose low 16 bits are 0x8000, so a v more than 128 ulps from one
          // (and inside [2^-90, 2^126), where neither underflow nor the clamps play a part)
          // rounds as the exact least-squares quotient does. Otherwise (about 0.4% of the
          // blocks, and every empty block) the block sums are taken again in binary64.
          float2 num2 = make_float2(0.f, 0.f), den2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            const float2 qc = mul2(q[p], cc[p]);
            num2 = fma2(w[p], qc, num2);
            den2 = fma2(qc, qc, den2);
          }
          float num = num2.x + num2.y, den = den2.x + den2.y;
#pragma unroll
          for (int off = 1; off < LPB; off <<= 1) {
            num += __shfl_xor_sync(FULL, num, off);
            den += __shfl_xor_sync(FULL, den, off);
          }
          const float v = __fdiv_rn(num, den);
          const uint32_t lo = __float_as_uint(v) & 0xFFFFu;
          const bool sure = num >= 0x1p-90f && den >= 0x1p-90f && v >= 0x1p-90f &&
                            v < 0x1p126f && (lo + 128u - 0x8000u) > 256u;
          uint32_t code = project_code<SCALE>(v, s_t);
          if (__any_sync(FULL, !sure)) {
            double num64 = 0.0, den64 = 0.0;
#pragma unroll
            for (int p = 0; p < 8; ++p) {
              const double qcx = (double)q[p].x * (double)cc[p].x;
              const double qcy = (double)q[p].y * (double)cc[p].y;
              num64 = fma((double)w[p].x, qcx, num64);
              num64 = fma((double)w[p].y, qcy, num64);
              den64 = fma(qcx, qcx, den64);
              den64 = fma(qcy, qcy, den64);
            }
#pragma unroll
            for (int off = 1; off < LPB; off <<= 1) {
              num64 += __shfl_xor_sync(FULL, num64, off);
              den64 += __shfl_xor_sync(FULL, den64, off);
            }
            if (!sure)
              code = (den64 > 0.0) ? project_code<SCALE>(div64_to_f32(num64, den64), s_t)
                                   : sc.code;
          }
          sc = dec(code);
        } else {
          float2 num2 = make_float2(0.f, 0.f), den2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            const float2 qc = mul2(q[p], cc[p]);
            num2 = fma2(w[p], qc, num2);
            den2 = fma2(qc, qc, den2);
          }
          float num = num2.x + num2.y, den = den2.x + den2.y;
#pragma unroll
          for (int off = 1; off < LPB; off <<= 1) {
            num += __shfl_xor_sync(FULL, num, off);
            den += __shfl_xor_sync(FULL, den, off);
          }
          sc = project_scale_ls<SCALE>(num, den, s_t, tbl, sc.code);
        }
      }
      if (lib == 0) {
        set_code(k, sc.code);
        if constexpr (EXT && ITER) {
          if (qch) set_pcode(k, old_code);
        }
      }

      // c-step partial sums with the new r
      const float2 rr = make_float2(sc.r, sc.r);
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const float2 qr = mul2(q[p], rr);
        accN[p] = fma2(w[p], qr, accN[p]);
        accD[p] = fma2(qr, qr, accD[p]);
        if constexpr (INIT) accW2 = fma2(w[p], w[p], accW2);
      }

      if constexpr (EMIT) {
        if (row < m) {
          if constexpr (BYTE_CODES) {
            uint8_t* qp = M.q_packed + (int64_t)row * qpitch + col0 + s * 16;
            *reinterpret_cast<uint4*>(qp) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
          } else {
            uint8_t* qp = M.q_packed + (int64_t)row * qpitch + (col0 + s * 16) / 2;
            *reinterpret_cast<uint2*>(qp) = make_uint2(codes[0], codes[1]);
          }
          if (lib == 0) {
            const int64_t bi = (int64_t)row * nb + col0 / B + bl;
            M.r[bi] = sc.r;
            if constexpr (SCB == 2) reinterpret_cast<uint16_t*>(M.bscale)[bi] = (uint16_t)sc.code;
            else reinterpret_cast<uint8_t*>(M.bscale)[bi] = (uint8_t)sc.code;
          }
        }
      }
    };
    using N0 = std::integral_constant<int, 0>;
    using N1 = std::integral_constant<int, 1>;
    using N2 = std::integral_constant<int, 2>;
    if constexpr (SPLIT_ROWS) {
      const int kres = min(KS, RPT) - 1;   // row steps whose next row is resident
      int k = 0;
      for (; k < kres; ++k) step(k, N1{});
      // sweeps up to RPT - 2 lie wholly below m (only the last can be partial): with 32-byte
      // aligned rows, fetched with no per-row test (-2.9% on the 8B layer set)
      if (wide) {
        for (; k < RPT - 2; ++k) step(k, std::integral_constant<int, 4>{});
      }
      for (; k < RPT - 1; ++k) step(k, N2{});
      step(RPT - 1, N0{});
    } else {
      for (int k = 0; k < RPT; ++k) step(k, std::integral_constant<int, 3>{});
    }
    if (INIT && bad) atomicOr(L.err_word, ERRBIT_NONFINITE);

    // ---- Q-change sums of this pass: per warp (exact), summed by thread 0 below
    if (qch) {
      double qd = (double)accQd.x + (double)accQd.y, qp = (double)accQp.x + (double)accQp.y;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) {
        qd += __shfl_xor_sync(FULL, qd, off);
        qp += __shfl_xor_sync(FULL, qp, off);
      }
      if (lane == 0) {
        qred[2 * warp] = qd;
        qred[2 * warp + 1] = qp;
      }
    }

    // ---- iteration 0: ||W||^2 of the tile and (FUSE) the direct error sum, per warp
    if constexpr (INIT) {
      double w2 = (double)accW2.x + (double)accW2.y, e0 = (double)accE0.x + (double)accE0.y;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) {
        w2 += __shfl_xor_sync(FULL, w2, off);
        if constexpr (FUSE) e0 += __shfl_xor_sync(FULL, e0, off);
      }
      if (lane == 0) {
        wsqw[warp] = w2;
        if constexpr (FUSE) e0w[warp] = e0;
      }
    }

    // ---- column sums
    const double nd = column_totals(accN, accD);

    // ---- c-step (closed form) and this pass's error terms: warps 0..S-1, lanes 0..15
    if (tid < 32 * S) {
      const double Dj = __shfl_down_sync(FULL, nd, 16);
      double e = 0.0;
      if (lane < 16) {
        const int j = warp * 16 + lane;
        const double Nj = nd;
        float cj = cvec[j];
        if (ITER && qch) picvec[j] = icvec[j];   // 1/c of this pass's Q-step
        if (ITER && upd_c && Dj > 0.0) {
          cj = __fdiv_rn(__double2float_rn(Nj), __double2float_rn(Dj));
          cvec[j] = cj;
          icvec[j] = __frcp_rn(cj);
        }
        if (EMIT) M.c[col0 + j] = cj;
        // this column's part of ||W - W_hat||^2 beyond ||W_j||^2 (added once per tile)
        const double cd = (double)cj;
        e = cd * cd * Dj - 2.0 * cd * Nj;
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) e += __shfl_xor_sync(FULL, e, off);
      if (lane == 0) errw[warp] = e;
    }
    __syncthreads();
    if constexpr (ITER) load_c();
    if (tid == 0) {
      if constexpr (INIT) {
        double q2 = 0.0;
#pragma unroll
        for (int i = 0; i < NWARP; ++i) q2 += wsqw[i];
        wsq_tile = q2;
        M.ws_wsq[tile] = q2;
      }
      double e = wsq_tile;
#pragma unroll
      for (int i = 0; i < S; ++i) e += errw[i];
      M.ws_err[(int64_t)t * tiles + tile] = e;
      if constexpr (FUSE) {
        double e0 = 0.0;
#pragma unroll
        for (int i = 0; i < NWARP; ++i) e0 += e0w[i];
        M.ws_err[tile] = e0;                          // iteration 0
        if (qch) {
          M.ws_qch[2 * tile] = 0.0;                   // iteration 0: no change
          M.ws_qch[2 * tile + 1] = 0.0;
        }
      }
      if (qch) {
        double qd = 0.0, qp = 0.0;
#pragma unroll
        for (int i = 0; i < NWARP; ++i) {
          qd += qred[2 * i];
          qp += qred[2 * i + 1];
        }
        M.ws_qch[2 * ((int64_t)t * tiles + tile)] = qd;
        M.ws_qch[2 * ((int64_t)t * tiles + tile) + 1] = qp;
      }
    }
  };

  using Y = std::true_type;
  using N = std::false_type;
  if (T == 0) {
    pass(Y{}, Y{}, N{}, 0);                  // iteration 0 only
  } else if (T == 1) {
    pass(Y{}, Y{}, Y{}, 1);                  // iterations 0 and 1, emitted
  } else {
    pass(Y{}, N{}, Y{}, 1);                  // iterations 0 and 1
    for (int t = 2; t < T; ++t) pass(N{}, N{}, N{}, t);
    pass(N{}, Y{}, N{}, T);
  }
}

template <int ELEM, int SCALE, int LPB, int S, bool F32IN, bool EXT>
cudaError_t launch_one(const SolveLaunch& L, int count, const SolvePlan& p, cudaStream_t st) {
  auto kern = solve_kernel<ELEM, SCALE, LPB, S, F32IN, EXT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)p.smem);
  if (e != cudaSuccess) return e;
  timing_before(st);
  kern<<<dim3((unsigned)p.tiles, (unsigned)count, 1), SOLVE_NT, p.smem, st>>>(L);
  e = cudaGetLastError();
  timing_after(st);
  count_launches(1);
  return e;
}

// tile width 16*S, S a power of two from LPB (one format block) to 8
template <int ELEM, int SCALE, int LPB, bool F32IN, bool EXT>
cudaError_t launch_s(const SolveLaunch& L, int count, const SolvePlan& p, cudaStream_t st) {
  switch (p.S) {
    case 1:
      if constexpr (LPB <= 1) return launch_one<ELEM, SCALE, LPB, 1, F32IN, EXT>(L, count, p, st);
      break;
    case 2:
      if constexpr (LPB <= 2) return launch_one<ELEM, SCALE, LPB, 2, F32IN, EXT>(L, count, p, st);
      break;
    case 4:
      if constexpr (LPB <= 4) return launch_one<ELEM, SCALE, LPB, 4, F32IN, EXT>(L, count, p, st);
      break;
    case 8: return launch_one<ELEM, SCALE, LPB, 8, F32IN, EXT>(L, count, p, st);
    default: break;
  }
  return cudaErrorInvalidValue;
}

template <int ELEM, int SCALE, int LPB, bool EXT>
cudaError_t launch_dtype(const SolveLaunch& L, int count, int esize, const SolvePlan& p,
                         cudaStream_t st) {
  return esize == 4 ? launch_s<ELEM, SCALE, LPB, true, EXT>(L, count, p, st)
                    : launch_s<ELEM, SCALE, LPB, false, EXT>(L, count, p, st);
}

// the 4-bit formats (kind as in dq.h; INT4 group 64 or 128)
template <bool EXT>
cudaError_t launch_solve_formats(const SolveLaunch& L, int count, int kind, int group,
                                 int esize, const SolvePlan& p, cudaStream_t s) {
  switch (kind) {
    case 0:
      if (group == 64) return launch_dtype<ELEM_INT4, SCALE_BF16, 4, EXT>(L, count, esize, p, s);
      return launch_dtype<ELEM_INT4, SCALE_BF16, 8, EXT>(L, count, esize, p, s);
    case 1: return launch_dtype<ELEM_INT4, SCALE_E8M0, 2, EXT>(L, count, esize, p, s);
    case 2: return launch_dtype<ELEM_E2M1, SCALE_E8M0, 2, EXT>(L, count, esize, p, s);
    case 3: return launch_dtype<ELEM_E2M1, SCALE_E4M3, 1, EXT>(L, count, esize, p, s);
    default: return cudaErrorInvalidValue;
  }
}

// the 8-bit formats: INT8 (group 64 or 128, bf16 scales), MXINT8 (32, E8M0)
template <bool EXT>
cudaError_t launch_solve_formats8(const SolveLaunch& L, int count, int kind, int group,
                                  int esize, const SolvePlan& p, cudaStream_t s) {
  switch (kind) {
    case 4:
      if (group == 64) return launch_dtype<ELEM_INT8, SCALE_BF16, 4, EXT>(L, count, esize, p, s);
      return launch_dtype<ELEM_INT8, SCALE_BF16, 8, EXT>(L, count, esize, p, s);
    case 5: return launch_dtype<ELEM_INT8, SCALE_E8M0, 2, EXT>(L, count, esize, p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace
}  // namespace dq
