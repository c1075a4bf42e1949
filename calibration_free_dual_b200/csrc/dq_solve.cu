// dq_solve.cu — cluster-resident dual-scale BCD solve (sm_100a).
//
// Method: DualQuant ("DualQuant: Dual-scale Calibration-free Weight-and-Activation
// Quantization for LLMs", Abstract): W ~ diag(r) Q diag(c) fitted by block coordinate
// descent, every block updated in closed form; the quantizer is a black box and the scales
// are projected onto the format's admissible set after each update (acceptodds.com
// abstract of the same paper); the normalised-MSE trace of Figure 2 (b).
//
// B200 design. With r per (row, B-column block) and c per column, every step couples only
// columns of one block (r-step) or rows of one column (c-step), so the solve decomposes
// exactly into independent B-column strips. One thread-block cluster owns one tile of
// TN = 16*S columns (whole blocks) and splits its m rows over K CTAs; each CTA copies its
// rows x TN slab of W into shared memory once and runs every BCD iteration from there, so W
// crosses HBM once per solve instead of once per iteration. Per iteration:
//   * each thread owns one 16-column segment of a set of rows; LPB = B/16 neighbouring
//     lanes share one block and combine its r-step sums with xor shuffles;
//   * Q-, r- and c-step run per row in registers with packed fp32x2 arithmetic
//     (FMUL2/FFMA2) and the E2M1/E4M3 cvt instructions;
//   * per-column sums N_j, D_j: transposed warp reduction (fp32), cross-warp sum (fp64),
//     then every CTA of the cluster sums the K per-CTA partials from distributed shared
//     memory in rank order (fp64), so all CTAs derive bit-identical c_j;
//   * one cluster barrier per iteration (double-buffered partial slots), no spin-waits.
#include <cooperative_groups.h>

#include <mutex>
#include <type_traits>
#include <utility>
#include <vector>

#include "dq_device.cuh"
#include "dq_internal.h"

namespace cg = cooperative_groups;

namespace dq {
namespace {

constexpr unsigned FULL = 0xFFFFFFFFu;

// 16-byte chunk position of chunk h of piece P (the SEG columns one thread owns in one row;
// row-major [R][TN] tile, pieces of CPP chunks). The 8 lanes of a quarter warp read 8
// consecutive pieces; the swizzle spreads them over the 8 bank groups.
template <int CPP>
__device__ __forceinline__ int chunk_pos(int P, int h) {
  if constexpr (CPP == 1) return P;
  else if constexpr (CPP == 2) return 2 * P + (h ^ ((P >> 2) & 1));
  else return 4 * P + (h ^ ((P >> 1) & 3));
}

template <int SEG, int ESZ>
__device__ __forceinline__ void load_piece(const unsigned char* Wsm, int P, float2 (&w)[SEG / 2]) {
  constexpr int CPP = SEG * ESZ / 16;
  const uint4* base = reinterpret_cast<const uint4*>(Wsm);
#pragma unroll
  for (int h = 0; h < CPP; ++h) {
    const uint4 v = base[chunk_pos<CPP>(P, h)];
    if constexpr (ESZ == 2) {
      w[4 * h + 0] = bf16x2_to_f2(v.x);
      w[4 * h + 1] = bf16x2_to_f2(v.y);
      w[4 * h + 2] = bf16x2_to_f2(v.z);
      w[4 * h + 3] = bf16x2_to_f2(v.w);
    } else {
      w[2 * h + 0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
      w[2 * h + 1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
    }
  }
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// Butterfly reduction of an NV-value vector over the 32/S lanes sharing segment
// s = lane % S. Lane L ends with NV*S/32 consecutive values starting at (L - s)*NV/32
// (fixed order: deterministic).
template <int S, int NV>
__device__ __forceinline__ void transpose_reduce(float (&v)[NV], int lane) {
  int cnt = NV;
#pragma unroll
  for (int off = 16; off >= S; off >>= 1) {
    const int half = cnt >> 1;
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < NV / 2; ++i) {
      if (i < half) {
        const float send = upper ? v[i] : v[i + half];
        const float keep = upper ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(FULL, send, off);
      }
    }
    cnt = half;
  }
}

// One CTA: rows [rank*R, rank*R + R) of the column tile [tile*TN, tile*TN + TN) of matrix
// blockIdx.y. Threads own SEG-column pieces of rows; LPB lanes share one format block.
template <int ELEM, int SCALE, int SEG, int LPB, int S, bool F32IN>
__global__ void __launch_bounds__(SOLVE_NT, 2)
solve_kernel(const __grid_constant__ SolveLaunch L) {
  constexpr int NT = SOLVE_NT, NWARP = NT / 32, TN = SEG * S, NBLK = S / LPB, B = SEG * LPB;
  constexpr int NG = NT / S;            // rows covered by one pass of all threads
  constexpr int NP = SEG / 2;           // float2 pairs per piece
  constexpr int NV = 2 * SEG;           // per-thread column sums (N, D) of one pass
  constexpr int VPL = NV * S / 32;      // reduced values per lane
  constexpr int ESZ = F32IN ? 4 : 2;
  constexpr int CPP = SEG * ESZ / 16;   // 16-byte chunks per piece
  constexpr int SCB = (SCALE == SCALE_BF16) ? 2 : 1;
  constexpr float QMAX = (ELEM == ELEM_INT4) ? 7.0f : 6.0f;
  static_assert(NBLK * LPB == S && S >= 1 && S <= 8 && (SEG == 8 || SEG == 16), "tile shape");

  cg::cluster_group cluster = cg::this_cluster();
  const int K = L.K, R = L.R, m = L.m, n = L.n, T = L.T, tiles = L.tiles;
  const int rank = (int)cluster.block_rank();
  const int row0 = rank * R;
  const int Rc = max(0, min(R, m - row0));
  const int tile = blockIdx.x / K;
  const SolveMat& M = L.mats[blockIdx.y];
  const int col0 = tile * TN;
  const int nb = n / B;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = tid % S, g = tid / S, bl = s / LPB, lib = s % LPB;

  extern __shared__ __align__(128) unsigned char smem[];
  const SolveSmem lay = solve_smem(R, S, LPB, ESZ, SCB, K, SEG);
  unsigned char* Wsm = smem + lay.w;
  void* codes_v = smem + lay.codes;
  float2* tbl = reinterpret_cast<float2*>(smem + lay.tbl);
  float* cvec = reinterpret_cast<float*>(smem + lay.cvec);
  float* icvec = reinterpret_cast<float*>(smem + lay.icvec);
  float* red = reinterpret_cast<float*>(smem + lay.red);
  double* slot = reinterpret_cast<double*>(smem + lay.slot);
  double* colsum = reinterpret_cast<double*>(smem + lay.colsum);

  auto code_at = [&](int row) -> uint32_t {
    if constexpr (SCB == 2) return reinterpret_cast<uint16_t*>(codes_v)[row * NBLK + bl];
    else return reinterpret_cast<uint8_t*>(codes_v)[row * NBLK + bl];
  };
  auto set_code = [&](int row, uint32_t code) {
    if constexpr (SCB == 2) reinterpret_cast<uint16_t*>(codes_v)[row * NBLK + bl] = (uint16_t)code;
    else reinterpret_cast<uint8_t*>(codes_v)[row * NBLK + bl] = (uint8_t)code;
  };

  // ---- tensor scale (NVFP4) and the code -> (r, 1/r) table
  float s_t = 1.0f;
  if constexpr (SCALE == SCALE_E4M3) {
    s_t = nvfp4_tensor_scale(__uint_as_float(*M.amax_bits));
    if (tid < 128) {
      const uint32_t code = (tid == 0 || tid == 127) ? 1u : (uint32_t)tid;
      const float r = __fmul_rn(s_t, e4m3_decode(code));
      tbl[tid] = make_float2(r, __frcp_rn(r));
    }
    if (tile == 0 && rank == 0 && tid == 0 && M.tensor_scale != nullptr) *M.tensor_scale = s_t;
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

  // ---- copy this CTA's rows x TN slab of W into shared memory (the only read of W)
  {
    constexpr int CH = TN * ESZ / 16;      // 16-byte chunks per row
    const char* gW = reinterpret_cast<const char*>(M.W);
    const int64_t ldw = M.ldw;
    uint4* dst = reinterpret_cast<uint4*>(Wsm);
    bool bad = false;
#pragma unroll 4
    for (int ch = tid; ch < Rc * CH; ch += NT) {
      const int row = ch / CH, part = ch % CH;
      const uint4 v = ldg_stream(gW + ((int64_t)(row0 + row) * ldw + col0) * ESZ + part * 16);
      if constexpr (ESZ == 2) {
        bad |= bf16x2_nonfinite(v.x) | bf16x2_nonfinite(v.y) | bf16x2_nonfinite(v.z) |
               bf16x2_nonfinite(v.w);
      } else {
        bad |= !isfinite(__uint_as_float(v.x)) | !isfinite(__uint_as_float(v.y)) |
               !isfinite(__uint_as_float(v.z)) | !isfinite(__uint_as_float(v.w));
      }
      dst[chunk_pos<CPP>(row * S + part / CPP, part % CPP)] = v;
    }
    if (bad) atomicOr(L.err_word, ERRBIT_NONFINITE);
  }
  __syncthreads();

  float2 cc[NP], ic[NP];
  auto load_c = [&]() {
    const float4* cv = reinterpret_cast<const float4*>(cvec + s * SEG);
    const float4* iv = reinterpret_cast<const float4*>(icvec + s * SEG);
#pragma unroll
    for (int h = 0; h < SEG / 4; ++h) {
      const float4 a = cv[h], b = iv[h];
      cc[2 * h] = make_float2(a.x, a.y);
      cc[2 * h + 1] = make_float2(a.z, a.w);
      ic[2 * h] = make_float2(b.x, b.y);
      ic[2 * h + 1] = make_float2(b.z, b.w);
    }
  };
  load_c();

  const int RPT = (Rc + NG - 1) / NG;        // uniform within the CTA (shuffles below)
  const int nh = n >> 1;

  // One pass over the CTA's rows. INIT: iteration 0 (scales from absmax or r0, c = c0);
  // otherwise one BCD iteration (Q-step, r-step + projection, c-step sums). EMIT: the
  // returned state is written.
  auto pass = [&](auto init_tag, auto emit_tag, const int t) {
    constexpr bool INIT = decltype(init_tag)::value;
    constexpr bool EMIT = decltype(emit_tag)::value;
    float2 accN[NP], accD[NP], accS[INIT ? NP : 1];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      accN[p] = make_float2(0.f, 0.f);
      accD[p] = make_float2(0.f, 0.f);
      if constexpr (INIT) accS[p] = make_float2(0.f, 0.f);
    }

    for (int k = 0; k < RPT; ++k) {
      const int row = g + k * NG;
      const bool valid = row < Rc;
      float2 w[NP];
      if (valid) {
        load_piece<SEG, ESZ>(Wsm, row * S + s, w);
      } else {
#pragma unroll
        for (int p = 0; p < NP; ++p) w[p] = make_float2(0.f, 0.f);
      }

      ScaleVal sc;
      if constexpr (INIT) {
        float a = 0.0f;
#pragma unroll
        for (int p = 0; p < NP; ++p) a = fmaxf(a, fmaxf(fabsf(w[p].x), fabsf(w[p].y)));
#pragma unroll
        for (int off = 1; off < LPB; off <<= 1) a = fmaxf(a, __shfl_xor_sync(FULL, a, off));
        float v;
        if (M.r0 != nullptr) {
          v = valid ? M.r0[(int64_t)(row0 + row) * nb + col0 / B + bl] : 1.0f;
        } else {
          v = (a > 0.0f) ? __fdiv_rn(a, QMAX) : 1.0f;
        }
        sc = project_scale<SCALE>(v, s_t, tbl);
      } else {
        sc = scale_decode<SCALE>(valid ? code_at(row) : (SCALE == SCALE_BF16 ? 0x3F80u : 127u),
                                 tbl);
      }

      // Q-step on the binary32 quotient fl32(fl32(w * 1/c) * 1/r)
      float2 q[NP];
      uint32_t codes[(NP + 3) / 4];
#pragma unroll
      for (int i = 0; i < (NP + 3) / 4; ++i) codes[i] = 0u;
      const float2 irr = make_float2(sc.ir, sc.ir);
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const uint32_t cb = quant2<ELEM>(mul2(mul2(w[p], ic[p]), irr), q[p]);
        if constexpr (EMIT) codes[p >> 2] |= cb << (8 * (p & 3));
      }

      if constexpr (!INIT) {
        // r-step: least squares over the block, then projection
        if constexpr (SCALE == SCALE_BF16) {
          // INT4's fine bf16 scale grid: block sums in binary64 keep projection decisions
          // on the exact least-squares quotient
          double num = 0.0, den = 0.0;
#pragma unroll
          for (int p = 0; p < NP; ++p) {
            const double qcx = (double)q[p].x * (double)cc[p].x;
            const double qcy = (double)q[p].y * (double)cc[p].y;
            num = fma((double)w[p].x, qcx, num);
            num = fma((double)w[p].y, qcy, num);
            den = fma(qcx, qcx, den);
            den = fma(qcy, qcy, den);
          }
#pragma unroll
          for (int off = 1; off < LPB; off <<= 1) {
            num += __shfl_xor_sync(FULL, num, off);
            den += __shfl_xor_sync(FULL, den, off);
          }
          if (den > 0.0) sc = project_scale<SCALE>(__double2float_rn(num / den), s_t, tbl);
        } else {
          float2 num2 = make_float2(0.f, 0.f), den2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int p = 0; p < NP; ++p) {
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
          if (den > 0.0f) sc = project_scale_ls<SCALE>(num, den, s_t, tbl);
        }
      }
      if (valid && lib == 0) set_code(row, sc.code);

      // c-step partial sums with the new r
      const float2 rr = make_float2(sc.r, sc.r);
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const float2 qr = mul2(q[p], rr);
        accN[p] = fma2(w[p], qr, accN[p]);
        accD[p] = fma2(qr, qr, accD[p]);
        if constexpr (INIT) accS[p] = fma2(w[p], w[p], accS[p]);
      }

      if constexpr (EMIT) {
        if (valid) {
          uint8_t* qp = M.q_packed + (int64_t)(row0 + row) * nh + (col0 + s * SEG) / 2;
          if constexpr (NP == 8) *reinterpret_cast<uint2*>(qp) = make_uint2(codes[0], codes[1]);
          else *reinterpret_cast<uint32_t*>(qp) = codes[0];
          if (lib == 0) {
            const int64_t bi = (int64_t)(row0 + row) * nb + col0 / B + bl;
            M.r[bi] = sc.r;
            if constexpr (SCB == 2) reinterpret_cast<uint16_t*>(M.bscale)[bi] = (uint16_t)sc.code;
            else reinterpret_cast<uint8_t*>(M.bscale)[bi] = (uint8_t)sc.code;
          }
        }
      }
    }

    // ---- per-column sums: warp (fp32) -> CTA (fp64) -> cluster (fp64, rank order)
    const int buf = t & 1;
    double* bufslot = slot + buf * K * 2 * NV * S;      // [K ranks][2 NV S] of this iteration
    {
      float v[NV];
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        v[2 * p] = accN[p].x;
        v[2 * p + 1] = accN[p].y;
        v[SEG + 2 * p] = accD[p].x;
        v[SEG + 2 * p + 1] = accD[p].y;
      }
      transpose_reduce<S, NV>(v, lane);
#pragma unroll
      for (int i = 0; i < VPL; ++i) red[(warp * S + s) * NV + (lane - s) * NV / 32 + i] = v[i];
      if constexpr (INIT) {
        float u[NV];
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          u[2 * p] = accS[p].x;
          u[2 * p + 1] = accS[p].y;
          u[SEG + 2 * p] = 0.f;
          u[SEG + 2 * p + 1] = 0.f;
        }
        transpose_reduce<S, NV>(u, lane);
#pragma unroll
        for (int i = 0; i < VPL; ++i)
          red[NWARP * S * NV + (warp * S + s) * NV + (lane - s) * NV / 32 + i] = u[i];
      }
    }
    __syncthreads();
    if (tid < NV * S) {
      double acc = 0.0, acs = 0.0;
#pragma unroll
      for (int wp = 0; wp < NWARP; ++wp) acc += (double)red[wp * S * NV + tid];
      if constexpr (INIT) {
#pragma unroll
        for (int wp = 0; wp < NWARP; ++wp) acs += (double)red[NWARP * S * NV + wp * S * NV + tid];
      }
      // push this CTA's partial into row `rank` of every cluster peer's buffer
#pragma unroll
      for (int rk = 0; rk < SOLVE_MAXK; ++rk) {
        if (rk < K) {
          double* dst = cluster.map_shared_rank(bufslot, rk) + rank * 2 * NV * S;
          dst[tid] = acc;
          if constexpr (INIT) dst[NV * S + tid] = acs;
        }
      }
    }
    cluster.sync();

    // warp 0: per-column totals over the cluster (rank order), new c, error terms
    double e = 0.0, q2 = 0.0;
    if (warp == 0) {
#pragma unroll
      for (int jj = 0; jj < (TN + 31) / 32; ++jj) {
        const int j = lane + 32 * jj;
        if (j < TN) {
          const int sj = j / SEG, ej = j % SEG;
          double Nj = 0.0, Dj = 0.0, Sj = 0.0;
#pragma unroll
          for (int rk = 0; rk < SOLVE_MAXK; ++rk) {
            if (rk < K) {
              const double* rs = bufslot + rk * 2 * NV * S;
              Nj += rs[sj * NV + ej];
              Dj += rs[sj * NV + SEG + ej];
              if constexpr (INIT) Sj += rs[NV * S + sj * NV + ej];
            }
          }
          if constexpr (INIT) colsum[j] = Sj;
          else Sj = colsum[j];
          float cj = cvec[j];
          if (!INIT && Dj > 0.0) {
            cj = __fdiv_rn(__double2float_rn(Nj), __double2float_rn(Dj));
            cvec[j] = cj;
            icvec[j] = __frcp_rn(cj);
          }
          const double cd = (double)cj;
          e += Sj - 2.0 * cd * Nj + cd * cd * Dj;
          if constexpr (INIT) q2 += Sj;
          if (EMIT && rank == 0) M.c[col0 + j] = cj;
        }
      }
    }
    __syncthreads();
    if constexpr (!INIT) load_c();
    // trace terms of this tile (rank 0), off the other warps' critical path
    if (warp == 0 && rank == 0) {
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) {
        e += __shfl_xor_sync(FULL, e, off);
        if constexpr (INIT) q2 += __shfl_xor_sync(FULL, q2, off);
      }
      if (lane == 0) {
        M.ws_err[(int64_t)t * tiles + tile] = e;
        if constexpr (INIT) M.ws_wsq[tile] = q2;
      }
    }
  };

  if (T == 0) {
    pass(std::true_type{}, std::true_type{}, 0);
  } else {
    pass(std::true_type{}, std::false_type{}, 0);
    for (int t = 1; t < T; ++t) pass(std::false_type{}, std::false_type{}, t);
    pass(std::false_type{}, std::true_type{}, T);
  }

  // every peer has finished writing into and reading from this CTA's buffers
  cluster.sync();
}

// ----------------------------------------------------------------------------- amax
__global__ void solve_amax_kernel(const __grid_constant__ SolveLaunch L, int esize) {
  const SolveMat& M = L.mats[blockIdx.y];
  const int64_t rows = L.m, n = L.n, ldw = M.ldw;
  const int64_t cpr = n * esize / 16;                 // 16-byte chunks per row
  const int64_t total = rows * cpr;
  const char* base = reinterpret_cast<const char*>(M.W);
  float a = 0.0f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / cpr, part = i % cpr;
    const uint4 v = ldg_stream(base + row * ldw * esize + part * 16);
    if (esize == 2) {
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = bf16x2_to_f2(u[k]);
        a = fmaxf(a, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    } else {
      a = fmaxf(a, fmaxf(fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y))),
                         fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w)))));
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(FULL, a, off));
  if ((threadIdx.x & 31) == 0 && a > 0.0f) atomicMax(M.amax_bits, __float_as_uint(a));
}

// ------------------------------------------------------------------------- finalize
struct FinalizeArgs {
  double* mse[SOLVE_MAXMATS];
  double* err[SOLVE_MAXMATS];
  double* wsq[SOLVE_MAXMATS];
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
}

// Cluster size for a shape: among K >= the smallest that fits, the one with the most CTAs
// resident at once (cluster placement inside a GPC makes some sizes pack worse), ties to the
// smaller K; rows per CTA stay >= 32 once K exceeds the minimum. Depends on the shape and the
// device only, so results do not depend on how many matrices share a launch.
template <typename Kern>
SolvePlan choose_cluster(Kern kern, const SolvePlan& base, int m, int esize, int LPB, int scb) {
  struct Key { const void* k; int m, tiles; size_t smem; int dev; };
  static std::mutex mu;
  static std::vector<std::pair<Key, SolvePlan>> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const Key key{reinterpret_cast<const void*>(kern), m, base.tiles, base.smem, dev};
  {
    std::lock_guard<std::mutex> lk(mu);
    for (auto& e : cache)
      if (e.first.k == key.k && e.first.m == m && e.first.tiles == key.tiles &&
          e.first.smem == key.smem && e.first.dev == dev)
        return e.second;
  }
  SolvePlan best = base;
  int64_t best_ctas = -1;
  for (int K = base.K; K <= SOLVE_MAXK; ++K) {
    const int R = (m + K - 1) / K;
    if (K > base.K && R < 32) break;
    const SolveSmem l = solve_smem(R, base.S, LPB, esize, scb, K, SOLVE_SEG);
    if (l.total > 227 * 1024) continue;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)l.total) !=
        cudaSuccess) {
      (void)cudaGetLastError();
      continue;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(K * base.tiles), 1, 1);
    cfg.blockDim = dim3(SOLVE_NT, 1, 1);
    cfg.dynamicSmemBytes = l.total;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)K;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) != cudaSuccess || active <= 0) {
      (void)cudaGetLastError();
      continue;
    }
    const int64_t ctas = (int64_t)K * std::min<int64_t>(active, base.tiles);
    if (ctas > best_ctas) {
      best_ctas = ctas;
      best.K = K;
      best.R = R;
      best.smem = l.total;
    }
  }
  std::lock_guard<std::mutex> lk(mu);
  cache.emplace_back(key, best);
  return best;
}

template <int ELEM, int SCALE, int LPB, int S, bool F32IN>
cudaError_t launch_one(const SolveLaunch& L0, int count, const SolvePlan& p0, cudaStream_t st) {
  auto kern = solve_kernel<ELEM, SCALE, SOLVE_SEG, LPB, S, F32IN>;
  constexpr int ESZ = F32IN ? 4 : 2;
  const SolvePlan p = choose_cluster(kern, p0, L0.m, ESZ, LPB, SCALE == SCALE_BF16 ? 2 : 1);
  SolveLaunch L = L0;
  L.K = p.K;
  L.R = p.R;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)p.smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.K * p.tiles), (unsigned)count, 1);
  cfg.blockDim = dim3(SOLVE_NT, 1, 1);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.K;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  timing_before(st);
  e = cudaLaunchKernelEx(&cfg, kern, L);
  timing_after(st);
  count_launches(1);
  return e;
}

template <int ELEM, int SCALE, int LPB, int S>
cudaError_t launch_dtype(const SolveLaunch& L, int count, int esize, const SolvePlan& p,
                         cudaStream_t st) {
  return esize == 4 ? launch_one<ELEM, SCALE, LPB, S, true>(L, count, p, st)
                    : launch_one<ELEM, SCALE, LPB, S, false>(L, count, p, st);
}

}  // namespace

bool plan_solve(int64_t m, int64_t n, int kind, int group, int esize, int64_t ctas_hint,
                SolvePlan* p) {
  (void)ctas_hint;
  const int B = fmt_block(kind, group);
  if (B == 0 || m <= 0 || n <= 0 || n % B) return false;
  const int LPB = B / SOLVE_SEG;
  // the tile is one format block wide (NVFP4: 16, MX: 32, INT4: the group)
  const int S = LPB;
  const int scb = kind == 0 ? 2 : 1;
  // smallest cluster whose CTAs fit two per SM (the register limit), else one
  const size_t budgets[2] = {SOLVE_SMEM_2PERSM, SOLVE_SMEM_1PERSM};
  for (size_t budget : budgets) {
    for (int K = 1; K <= SOLVE_MAXK; ++K) {
      const int R = (int)((m + K - 1) / K);
      const SolveSmem l = solve_smem(R, S, LPB, esize, scb, K, SOLVE_SEG);
      if (l.total <= budget) {
        p->S = S;
        p->K = K;
        p->R = R;
        p->tiles = (int)(n / (SOLVE_SEG * S));
        p->smem = l.total;
        return true;
      }
    }
  }
  return false;
}

cudaError_t launch_solve(const SolveLaunch& L, int count, int kind, int group, int esize,
                         const SolvePlan& p, cudaStream_t s) {
  switch (kind) {
    case 0:
      if (group == 64) return launch_dtype<ELEM_INT4, SCALE_BF16, 4, 4>(L, count, esize, p, s);
      return launch_dtype<ELEM_INT4, SCALE_BF16, 8, 8>(L, count, esize, p, s);
    case 1: return launch_dtype<ELEM_INT4, SCALE_E8M0, 2, 2>(L, count, esize, p, s);
    case 2: return launch_dtype<ELEM_E2M1, SCALE_E8M0, 2, 2>(L, count, esize, p, s);
    case 3: return launch_dtype<ELEM_E2M1, SCALE_E4M3, 1, 1>(L, count, esize, p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_solve_amax(const SolveLaunch& L, int count, int esize, cudaStream_t s) {
  const int64_t chunks = (int64_t)L.m * L.n * esize / 16;
  int blocks = (int)std::min<int64_t>((chunks + 255) / 256, 1184);
  if (blocks < 1) blocks = 1;
  solve_amax_kernel<<<dim3(blocks, count), 256, 0, s>>>(L, esize);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_finalize(double* const* mse, double* const* ws_err, double* const* ws_wsq,
                            const int* tiles, int count, int T, cudaStream_t s) {
  for (int base = 0; base < count; base += SOLVE_MAXMATS) {
    FinalizeArgs A = {};
    const int c = std::min(SOLVE_MAXMATS, count - base);
    for (int i = 0; i < c; ++i) {
      A.mse[i] = mse[base + i];
      A.err[i] = ws_err[base + i];
      A.wsq[i] = ws_wsq[base + i];
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
