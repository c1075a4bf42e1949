// dq_internal.h — launch descriptors shared by the host API and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>   // CUtensorMap (the encoder is fetched from the driver at run time)
#include <cuda_runtime.h>

namespace dq {

constexpr int SOLVE_NT = 512;          // threads per CTA of the solve kernel (one CTA per SM)
constexpr int SOLVE_MAXMATS = 64;      // matrices per solve launch (descriptors by value)
constexpr size_t SOLVE_SMEM_MAX = 227 * 1024;   // dynamic shared memory of one CTA

struct SolveMat {
  const void* W;
  int64_t ldw;
  const float* r0;
  const float* c0;
  uint8_t* q_packed;
  float* r;
  float* c;
  void* bscale;
  float* tensor_scale;
  double* ws_err;              // [(T+1) * tiles] per-iteration partial errors
  double* ws_wsq;              // [tiles] partial ||W||^2
  double* ws_qch;              // [(T+1) * tiles * 2] Q-change partials (sum dq^2, sum q^2)
  unsigned* amax_bits;         // NVFP4: amax |W| as float bits (zeroed before the pre-pass)
};

struct SolveLaunch {
  int m, n, T;
  int R;                       // rows of each column tile kept in shared memory
  int tiles, count;
  int wide;                    // every W base and row pitch 32-byte aligned (256-bit loads)
  int upd_r, upd_c;            // extended kernel: which scales the iterations update
  int qch;                     // extended kernel: record the Q-change trace
  unsigned* err_word;
  SolveMat mats[SOLVE_MAXMATS];
  // tma != 0: wmap[i] maps matrix i's W as [m][n/16][16] (rows, 16-column pieces, columns)
  // with boxes of {16, S, solve_box_rows(S)} and the 32-byte (bf16) or 64-byte (fp32)
  // swizzle, and the kernel copies its resident rows with the tensor memory accelerator
  int tma;
  CUtensorMap wmap[SOLVE_MAXMATS];
};

// rows per tensor-map box of the solve's resident-row copy: one sweep (512/S rows), at most
// the 256 a box dimension allows
__host__ __device__ constexpr int solve_box_rows(int S) { return SOLVE_NT / S < 256 ? SOLVE_NT / S : 256; }

// the solve's W tensor map (see SolveLaunch::wmap); false when the driver's encoder is missing
// or refuses the shape
bool make_w_map(CUtensorMap* map, const void* W, int64_t m, int64_t n, int64_t ldw, int esize,
                int S);

struct SolvePlan {
  int S;        // 16-column pieces per CTA tile (tile width TN = 16*S)
  int R;        // rows of the tile resident in shared memory (the rest stream from L2)
  int tiles;    // column tiles per matrix (n / TN)
  size_t smem;  // dynamic shared memory per CTA
};

// Shared-memory carve-up of a solve CTA (same arithmetic on host and device): the resident
// rows of W (R, a whole number of sweeps), the scale code of every (row, block) of the tile
// with the rows rounded up to whole sweeps, the E4M3 table, c and 1/c,
// the per-warp column partials and the per-warp fp64 error sums; with the Q-change trace
// also the previous iteration's scale codes, its 1/c and per-warp Q-change sums.
struct SolveSmem {
  size_t w, codes, tbl, cvec, icvec, red, cols, pcodes, picvec, qred, bar, total;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline SolveSmem solve_smem(int m, int R, int S, int LPB, int esize,
                                                 int scb, bool qch) {
  const int TN = 16 * S, NBLK = S / LPB, NWARP = SOLVE_NT / 32, NG = SOLVE_NT / S;
  const size_t mpad = ((size_t)m + NG - 1) / NG * NG;    // rows rounded up to whole sweeps
  SolveSmem l;
  size_t off = 0;
  l.w = off;      off = align_up(off + (size_t)R * TN * esize, 128);
  l.codes = off;  off = align_up(off + mpad * NBLK * scb, 16);
  l.tbl = off;    off = align_up(off + 128 * 8, 16);
  l.cvec = off;   off = align_up(off + TN * 4, 16);
  l.icvec = off;  off = align_up(off + TN * 4, 16);
  l.red = off;    off = align_up(off + (size_t)NWARP * S * 32 * 4, 16);
  l.cols = off;   off = align_up(off + (size_t)4 * TN * 8, 16);
  l.pcodes = off; if (qch) off = align_up(off + mpad * NBLK * scb, 16);
  l.picvec = off; if (qch) off = align_up(off + TN * 4, 16);
  l.qred = off;   if (qch) off = align_up(off + (size_t)NWARP * 2 * 8, 16);
  l.bar = off;    off = align_up(off + 8, 16);           // the resident-row copy's mbarrier
  l.total = off;
  return l;
}

// format helpers (kind as in dq.h: INT4, MXINT4, MXFP4, NVFP4, INT8, MXINT8)
inline int fmt_block(int kind, int group) {
  switch (kind) {
    case 0: case 4: return (group == 64 || group == 128) ? group : 0;
    case 1: case 2: case 5: return group == 32 ? 32 : 0;
    case 3: return group == 16 ? 16 : 0;
    default: return 0;
  }
}
inline int fmt_scale_bytes(int kind) { return (kind == 0 || kind == 4) ? 2 : 1; }   // bf16: 2
inline int fmt_elem_bits(int kind) { return kind >= 4 ? 8 : 4; }

// measurement hooks (dq_api.cu)
void count_launches(int n);
void timing_before(cudaStream_t s);
void timing_after(cudaStream_t s);

// qch: the plan leaves room for the Q-change trace (its tile width, hence every result, is
// the same either way)
bool plan_solve(int64_t m, int64_t n, int kind, int group, int esize, bool qch, SolvePlan* p);
cudaError_t launch_solve(const SolveLaunch& L, int count, int kind, int group, int esize,
                         const SolvePlan& p, cudaStream_t s);
// the extended instantiation: update modes and the Q-change trace (L.upd_r, L.upd_c, L.qch)
cudaError_t launch_solve_ext(const SolveLaunch& L, int count, int kind, int group, int esize,
                             const SolvePlan& p, cudaStream_t s);
// the 8-bit formats (INT8, MXINT8), plain or extended
cudaError_t launch_solve_8bit(const SolveLaunch& L, int count, int kind, int group, int esize,
                              const SolvePlan& p, bool ext, cudaStream_t s);
cudaError_t launch_solve_8bit_ext(const SolveLaunch& L, int count, int kind, int group,
                                  int esize, const SolvePlan& p, cudaStream_t s);
cudaError_t launch_solve_amax(const SolveLaunch& L, int count, int esize, cudaStream_t s);
// qchange / ws_qch may be null (no Q-change trace)
cudaError_t launch_finalize(double* const* mse, double* const* ws_err, double* const* ws_wsq,
                            double* const* qchange, double* const* ws_qch, const int* tiles,
                            int count, int T, cudaStream_t s);

// NVFP4 activation pre-pass: at most this many CTAs, each writing its own maximum
constexpr int ACT_MAX_PARTS = 4096;

struct ActLaunch {
  const void* X;
  int64_t tokens, n, ldx;
  const float* c;
  uint8_t* x_packed;
  void* scales;
  float* tensor_scale;
  unsigned* partials;  // NVFP4: [ACT_MAX_PARTS] per-CTA amax of the pre-pass (float bits)
  unsigned* err_word;
  int sf_tc;          // NVFP4: scales in the tensor core's layout (see dq_gemm.h), else [tokens, n/16]
};
cudaError_t launch_act(const ActLaunch& A, int kind, int group, int esize, cudaStream_t s);

cudaError_t launch_encode(const float* x, int64_t count, int codec, void* codes,
                          cudaStream_t s);
cudaError_t launch_decode(const void* codes, int64_t count, int codec, float* x,
                          cudaStream_t s);

}  // namespace dq
