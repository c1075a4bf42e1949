// dq_api.cu — the extern "C" entry points declared in include/dq.h.
//
// Host side only: argument validation (before anything is queued), workspace carving,
// grouping of a layer set by matrix shape, and kernel launches. No allocation: every buffer,
// including the workspace, belongs to the caller.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "dq.h"
#include "dq_internal.h"
#include "dq_gemm.h"

namespace {

// Per-device error word raised by the kernels (non-finite input, bad warm start).
__device__ unsigned g_dq_err_word;

constexpr int MAX_DEVICES = 64;
std::mutex g_err_mu;
unsigned* g_err_ptr[MAX_DEVICES] = {};

dq_status err_word_ptr(unsigned** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return DQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (g_err_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dq_err_word) != cudaSuccess) return DQ_ERR_CUDA;
    g_err_ptr[dev] = static_cast<unsigned*>(p);
  }
  *out = g_err_ptr[dev];
  return DQ_OK;
}

int dtype_size(int32_t dt) { return dt == DQ_F32 ? 4 : (dt == DQ_BF16 ? 2 : 0); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t per_matrix_ws(int tiles, int iters, bool qch) {
  // ||W||^2 partials [tiles], error partials [(iters+1) * tiles], and with the Q-change
  // trace its partials [(iters+1) * tiles * 2]
  const size_t per = (size_t)(iters + 2) + (qch ? 2 * (size_t)(iters + 1) : 0);
  return dq::align_up(sizeof(double) * (size_t)tiles * per, 256);
}

// head of the workspace: one amax word per matrix (cleared by a single memset)
size_t amax_head(int64_t count) { return dq::align_up(sizeof(unsigned) * (size_t)count, 256); }

dq_status check_format(dq_format f) {
  if (f.kind < DQ_INT4 || f.kind > DQ_MXINT8) return DQ_ERR_DTYPE;
  if (dq::fmt_block(f.kind, f.group) == 0) return DQ_ERR_DTYPE;
  return DQ_OK;
}

dq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? DQ_OK : DQ_ERR_CUDA; }

// measurement hooks
std::atomic<int64_t> g_launches{0};
thread_local void* const* t_ev_start = nullptr;
thread_local void* const* t_ev_stop = nullptr;
thread_local int32_t t_ev_cap = 0;
thread_local int32_t t_ev_used = 0;

}  // namespace

namespace dq {
void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
void timing_before(cudaStream_t s) {
  if (t_ev_used < t_ev_cap) cudaEventRecord(static_cast<cudaEvent_t>(t_ev_start[t_ev_used]), s);
}
void timing_after(cudaStream_t s) {
  if (t_ev_used < t_ev_cap) {
    cudaEventRecord(static_cast<cudaEvent_t>(t_ev_stop[t_ev_used]), s);
    ++t_ev_used;
  }
}
}  // namespace dq

extern "C" {

const char* dq_status_string(int32_t s) {
  switch (s) {
    case DQ_OK: return "DQ_OK";
    case DQ_ERR_INVALID_ARG: return "DQ_ERR_INVALID_ARG";
    case DQ_ERR_SHAPE: return "DQ_ERR_SHAPE";
    case DQ_ERR_DTYPE: return "DQ_ERR_DTYPE";
    case DQ_ERR_WORKSPACE: return "DQ_ERR_WORKSPACE";
    case DQ_ERR_NONFINITE: return "DQ_ERR_NONFINITE";
    case DQ_ERR_TIMEOUT: return "DQ_ERR_TIMEOUT";
    case DQ_ERR_CUDA: return "DQ_ERR_CUDA";
    case DQ_ERR_UNSUPPORTED: return "DQ_ERR_UNSUPPORTED";
    default: return "DQ_ERR_UNKNOWN";
  }
}

int64_t dq_solve_max_rows(int64_t n, dq_format fmt, int32_t dtype) {
  if (check_format(fmt) != DQ_OK || dtype_size(dtype) == 0 || n <= 0) return 0;
  int64_t lo = 0, hi = 1 << 26;
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) / 2;
    dq::SolvePlan p;
    if (dq::plan_solve(mid, n, fmt.kind, fmt.group, dtype_size(dtype), false, &p)) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

size_t dq_solve_workspace_bytes_ex(int64_t count, const int64_t* m, const int64_t* n,
                                   dq_format fmt, int32_t iters,
                                   const dq_solve_options* options) {
  if (count <= 0 || m == nullptr || n == nullptr || iters < 0) return 0;
  if (check_format(fmt) != DQ_OK) return 0;
  const bool qch = options != nullptr && options->qchange != nullptr;
  size_t total = amax_head(count);
  for (int64_t i = 0; i < count; ++i) {
    dq::SolvePlan p;
    // a shape is supported if some input dtype fits
    if (!dq::plan_solve(m[i], n[i], fmt.kind, fmt.group, 2, qch, &p) &&
        !dq::plan_solve(m[i], n[i], fmt.kind, fmt.group, 4, qch, &p))
      return 0;
    // room for one tile per format block, the most tiles any plan uses
    total += per_matrix_ws((int)(n[i] / dq::fmt_block(fmt.kind, fmt.group)), iters, qch);
  }
  return total;
}

size_t dq_solve_workspace_bytes(int64_t count, const int64_t* m, const int64_t* n,
                                dq_format fmt, int32_t iters) {
  return dq_solve_workspace_bytes_ex(count, m, n, fmt, iters, nullptr);
}

dq_status dq_solve_batched_ex(const dq_matrix* mats, int64_t count, int32_t dtype,
                              dq_format fmt, int32_t iters, const dq_solve_options* options,
                              void* workspace, size_t workspace_bytes, void* stream) {
  if (mats == nullptr || count <= 0 || iters < 0 || iters > (1 << 20)) return DQ_ERR_INVALID_ARG;
  const int32_t update = options != nullptr ? options->update : DQ_UPDATE_BOTH;
  if (update != DQ_UPDATE_BOTH && update != DQ_UPDATE_ROW_ONLY && update != DQ_UPDATE_COL_ONLY)
    return DQ_ERR_INVALID_ARG;
  double* const* qchange = options != nullptr ? options->qchange : nullptr;
  const bool qch = qchange != nullptr;
  if (qch)
    for (int64_t i = 0; i < count; ++i)
      if (qchange[i] == nullptr) return DQ_ERR_INVALID_ARG;
  dq_status st = check_format(fmt);
  if (st != DQ_OK) return st;
  const int esize = dtype_size(dtype);
  if (esize == 0) return DQ_ERR_DTYPE;
  const int B = dq::fmt_block(fmt.kind, fmt.group);
  std::vector<int64_t> ms(count), ns(count);
  for (int64_t i = 0; i < count; ++i) {
    const dq_matrix& d = mats[i];
    if (d.m <= 0 || d.n <= 0 || d.ldw < d.n) return DQ_ERR_INVALID_ARG;
    if (d.n % B != 0) return DQ_ERR_SHAPE;
    if (d.m > INT32_MAX / 2 || d.n > INT32_MAX / 2) return DQ_ERR_SHAPE;
    if (d.W == nullptr || d.q_packed == nullptr || d.r == nullptr || d.c == nullptr ||
        d.block_scales == nullptr || d.mse_trace == nullptr)
      return DQ_ERR_INVALID_ARG;
    if (fmt.kind == DQ_NVFP4 && d.tensor_scale == nullptr) return DQ_ERR_INVALID_ARG;
    if (!aligned16(d.W) || (d.ldw * esize) % 16 != 0) return DQ_ERR_INVALID_ARG;
    // 4-bit codes are stored 8 bytes per thread, 8-bit codes 16
    const uintptr_t qalign = dq::fmt_elem_bits(fmt.kind) == 8 ? 15u : 7u;
    if ((reinterpret_cast<uintptr_t>(d.q_packed) & qalign) != 0) return DQ_ERR_INVALID_ARG;
    ms[i] = d.m;
    ns[i] = d.n;
  }
  const size_t need = dq_solve_workspace_bytes_ex(count, ms.data(), ns.data(), fmt, iters,
                                                  options);
  if (need == 0) return DQ_ERR_UNSUPPORTED;
  if (workspace == nullptr || workspace_bytes < need) return DQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return DQ_ERR_INVALID_ARG;

  unsigned* errp = nullptr;
  if ((st = err_word_ptr(&errp)) != DQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // carve the workspace per matrix
  struct Slot {
    dq::SolvePlan plan;
    unsigned* amax;
    double* wsq;
    double* err;
    double* qch;
  };
  std::vector<Slot> slots(count);
  char* ws = static_cast<char*>(workspace);
  size_t off = amax_head(count);
  if (fmt.kind == DQ_NVFP4) {
    if ((st = from_cuda(cudaMemsetAsync(ws, 0, sizeof(unsigned) * (size_t)count, s))) != DQ_OK)
      return st;
  }
  for (int64_t i = 0; i < count; ++i) {
    Slot& sl = slots[i];
    // the plan depends on the matrix shape only, so a matrix gets bit-identical results
    // whether it is solved alone or inside a layer set
    if (!dq::plan_solve(ms[i], ns[i], fmt.kind, fmt.group, esize, qch, &sl.plan))
      return DQ_ERR_UNSUPPORTED;
    const int tiles_max = (int)(ns[i] / B);
    sl.amax = reinterpret_cast<unsigned*>(ws) + i;
    sl.wsq = reinterpret_cast<double*>(ws + off);
    sl.err = sl.wsq + sl.plan.tiles;
    sl.qch = qch ? sl.err + (size_t)(iters + 1) * sl.plan.tiles : nullptr;
    off += per_matrix_ws(tiles_max, iters, qch);
  }

  // group by shape (order of first appearance), launch in chunks of SOLVE_MAXMATS
  std::vector<char> done(count, 0);
  for (int64_t i = 0; i < count; ++i) {
    if (done[i]) continue;
    std::vector<int64_t> grp;
    for (int64_t j = i; j < count; ++j)
      if (!done[j] && ms[j] == ms[i] && ns[j] == ns[i]) {
        grp.push_back(j);
        done[j] = 1;
      }
    const dq::SolvePlan& plan = slots[i].plan;
    for (size_t base = 0; base < grp.size(); base += dq::SOLVE_MAXMATS) {
      const int c = (int)std::min<size_t>(dq::SOLVE_MAXMATS, grp.size() - base);
      dq::SolveLaunch L;
      std::memset(&L, 0, sizeof(L));
      L.m = (int)ms[i];
      L.n = (int)ns[i];
      L.T = iters;
      L.R = plan.R;
      L.tiles = plan.tiles;
      L.count = c;
      L.wide = 1;
      L.upd_r = update != DQ_UPDATE_COL_ONLY;
      L.upd_c = update != DQ_UPDATE_ROW_ONLY;
      L.qch = qch;
      L.err_word = errp;
      L.tma = 1;     // cleared when a map cannot be made: the kernel then copies per thread
      for (int k = 0; k < c; ++k) {
        const int64_t idx = grp[base + k];
        const dq_matrix& d = mats[idx];
        dq::SolveMat& sm = L.mats[k];
        sm.W = d.W;
        sm.ldw = d.ldw;
        if ((reinterpret_cast<uintptr_t>(d.W) & 31u) != 0 || (d.ldw * esize) % 32 != 0)
          L.wide = 0;
        sm.r0 = d.r0;
        sm.c0 = d.c0;
        sm.q_packed = d.q_packed;
        sm.r = d.r;
        sm.c = d.c;
        sm.bscale = d.block_scales;
        sm.tensor_scale = d.tensor_scale;
        sm.ws_err = slots[idx].err;
        sm.ws_wsq = slots[idx].wsq;
        sm.ws_qch = slots[idx].qch;
        sm.amax_bits = slots[idx].amax;
        if (L.tma && !dq::make_w_map(&L.wmap[k], d.W, ms[i], ns[i], d.ldw, esize, plan.S))
          L.tma = 0;
      }
      if (fmt.kind == DQ_NVFP4) {
        if ((st = from_cuda(dq::launch_solve_amax(L, c, esize, s))) != DQ_OK) return st;
      }
      const bool ext = qch || update != DQ_UPDATE_BOTH;
      const cudaError_t e =
          dq::fmt_elem_bits(fmt.kind) == 8
              ? dq::launch_solve_8bit(L, c, fmt.kind, fmt.group, esize, plan, ext, s)
              : (ext ? dq::launch_solve_ext(L, c, fmt.kind, fmt.group, esize, plan, s)
                     : dq::launch_solve(L, c, fmt.kind, fmt.group, esize, plan, s));
      if ((st = from_cuda(e)) != DQ_OK) return st;
    }
  }
  std::vector<double*> mse(count), err(count), wsq(count), wqch(count);
  std::vector<int> tiles(count);
  for (int64_t i = 0; i < count; ++i) {
    mse[i] = mats[i].mse_trace;
    err[i] = slots[i].err;
    wsq[i] = slots[i].wsq;
    wqch[i] = slots[i].qch;
    tiles[i] = slots[i].plan.tiles;
  }
  return from_cuda(dq::launch_finalize(mse.data(), err.data(), wsq.data(), qchange,
                                       qch ? wqch.data() : nullptr, tiles.data(),
                                       (int)count, iters, s));
}

dq_status dq_solve_batched(const dq_matrix* mats, int64_t count, int32_t dtype, dq_format fmt,
                           int32_t iters, void* workspace, size_t workspace_bytes,
                           void* stream) {
  return dq_solve_batched_ex(mats, count, dtype, fmt, iters, nullptr, workspace,
                             workspace_bytes, stream);
}

dq_status dq_solve(const void* W, int32_t dtype, int64_t m, int64_t n, int64_t ldw,
                   dq_format fmt, int32_t iters, const float* r0, const float* c0,
                   uint8_t* q_packed, float* r, float* c, void* block_scales,
                   float* tensor_scale, double* mse_trace, void* workspace,
                   size_t workspace_bytes, void* stream) {
  dq_matrix d;
  d.W = W;
  d.m = m;
  d.n = n;
  d.ldw = ldw;
  d.r0 = r0;
  d.c0 = c0;
  d.q_packed = q_packed;
  d.r = r;
  d.c = c;
  d.block_scales = block_scales;
  d.tensor_scale = tensor_scale;
  d.mse_trace = mse_trace;
  return dq_solve_batched(&d, 1, dtype, fmt, iters, workspace, workspace_bytes, stream);
}

size_t dq_w4a4_gemm_workspace_bytes(int64_t T, int64_t N, int64_t K) {
  if (T <= 0 || N <= 0 || K <= 0 || K % 64 != 0) return 0;
  return dq::gemm_workspace_bytes(T, N, K);
}

dq_status dq_w4a4_gemm(const uint8_t* x_packed, const uint8_t* x_scales,
                       const float* x_tensor_scale, int64_t T, const uint8_t* w_packed,
                       const uint8_t* w_scales, const float* w_tensor_scale, int64_t N,
                       int64_t K, dq_format fmt, float* y, int64_t ldy, void* workspace,
                       size_t workspace_bytes, void* stream) {
  dq_status st = check_format(fmt);
  if (st != DQ_OK) return st;
  if (fmt.kind != DQ_NVFP4) return DQ_ERR_UNSUPPORTED;
  if (T <= 0 || N <= 0 || K <= 0 || ldy < N) return DQ_ERR_INVALID_ARG;
  if (K % 64 != 0) return DQ_ERR_SHAPE;
  if (T > ((int64_t)1 << 30) || N > ((int64_t)1 << 30) || K > ((int64_t)1 << 30))
    return DQ_ERR_SHAPE;
  if (x_packed == nullptr || x_scales == nullptr || x_tensor_scale == nullptr ||
      w_packed == nullptr || w_scales == nullptr || w_tensor_scale == nullptr || y == nullptr)
    return DQ_ERR_INVALID_ARG;
  if (!aligned16(x_packed) || !aligned16(w_packed)) return DQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x_scales) & 3u) || (reinterpret_cast<uintptr_t>(w_scales) & 3u) ||
      (reinterpret_cast<uintptr_t>(y) & 3u))
    return DQ_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < dq_w4a4_gemm_workspace_bytes(T, N, K))
    return DQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return DQ_ERR_INVALID_ARG;
  unsigned* errp = nullptr;
  if ((st = err_word_ptr(&errp)) != DQ_OK) return st;
  dq::GemmArgs A = {};
  A.xq = x_packed;
  A.xs = x_scales;
  A.xst = x_tensor_scale;
  A.wq = w_packed;
  A.ws = w_scales;
  A.wst = w_tensor_scale;
  A.y = y;
  A.T = T;
  A.N = N;
  A.K = K;
  A.ldy = ldy;
  A.err_word = errp;
  return from_cuda(dq::launch_w4a4_gemm(A, workspace, static_cast<cudaStream_t>(stream)));
}

size_t dq_act_quant_workspace_bytes(int64_t tokens, int64_t n, dq_format fmt) {
  if (tokens < 0 || n <= 0 || check_format(fmt) != DQ_OK) return 0;
  // NVFP4: one maximum per CTA of the amax pre-pass
  return fmt.kind == DQ_NVFP4 ? (size_t)4 * dq::ACT_MAX_PARTS : 256;
}

dq_status dq_act_quant(const void* X, int32_t dtype, int64_t tokens, int64_t n, int64_t ldx,
                       const float* c, dq_format fmt, uint8_t* x_packed, void* scales,
                       float* tensor_scale, void* workspace, size_t workspace_bytes,
                       void* stream) {
  dq_status st = check_format(fmt);
  if (st != DQ_OK) return st;
  const int esize = dtype_size(dtype);
  if (esize == 0) return DQ_ERR_DTYPE;
  if (tokens < 0 || n <= 0 || ldx < n) return DQ_ERR_INVALID_ARG;
  const int B = dq::fmt_block(fmt.kind, fmt.group);
  if (n % B != 0) return DQ_ERR_SHAPE;
  if (tokens == 0) return DQ_OK;
  if (X == nullptr || x_packed == nullptr || scales == nullptr) return DQ_ERR_INVALID_ARG;
  if (fmt.kind == DQ_NVFP4 && tensor_scale == nullptr) return DQ_ERR_INVALID_ARG;
  if (!aligned16(X) || (ldx * esize) % 16 != 0) return DQ_ERR_INVALID_ARG;
  if (c != nullptr && !aligned16(c)) return DQ_ERR_INVALID_ARG;
  const uintptr_t xalign = dq::fmt_elem_bits(fmt.kind) == 8 ? 7u : 3u;
  if ((reinterpret_cast<uintptr_t>(x_packed) & xalign) != 0) return DQ_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < dq_act_quant_workspace_bytes(tokens, n, fmt))
    return DQ_ERR_WORKSPACE;
  unsigned* errp = nullptr;
  if ((st = err_word_ptr(&errp)) != DQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  dq::ActLaunch A = {};
  A.X = X;
  A.tokens = tokens;
  A.n = n;
  A.ldx = ldx;
  A.c = c;
  A.x_packed = x_packed;
  A.scales = scales;
  A.tensor_scale = tensor_scale;
  A.partials = static_cast<unsigned*>(workspace);
  A.err_word = errp;
  return from_cuda(dq::launch_act(A, fmt.kind, fmt.group, esize, s));
}

// W4A4 linear layer: workspace = [activation tensor scale | per-CTA maxima of the amax
// pre-pass | activation codes | activation scale factors in the tensor core's layout |
// weight scale factors re-laid]
namespace {
struct LinearWs {
  size_t codes, sfa, sfb, total;
};
LinearWs linear_ws(int64_t T, int64_t N, int64_t K) {
  LinearWs l;
  const int64_t tpad = (T + 127) / 128 * 128;
  l.codes = 256 + (size_t)4 * dq::ACT_MAX_PARTS;
  l.sfa = dq::align_up(l.codes + (size_t)T * (size_t)(K / 2), 256);
  l.sfb = dq::align_up(l.sfa + (size_t)tpad * (size_t)(K / 16), 256);
  l.total = l.sfb + dq::gemm_workspace_bytes(T, N, K, true);
  return l;
}
}  // namespace

size_t dq_w4a4_linear_workspace_bytes(int64_t T, int64_t N, int64_t K, dq_format fmt) {
  if (check_format(fmt) != DQ_OK || fmt.kind != DQ_NVFP4) return 0;
  if (T <= 0 || N <= 0 || K <= 0 || K % 64 != 0) return 0;
  return linear_ws(T, N, K).total;
}

dq_status dq_w4a4_linear(const void* X, int32_t dtype, int64_t T, int64_t K, int64_t ldx,
                         const float* c, const uint8_t* w_packed, const uint8_t* w_scales,
                         const float* w_tensor_scale, int64_t N, dq_format fmt, float* y,
                         int64_t ldy, void* workspace, size_t workspace_bytes, void* stream) {
  dq_status st = check_format(fmt);
  if (st != DQ_OK) return st;
  if (fmt.kind != DQ_NVFP4) return DQ_ERR_UNSUPPORTED;
  const int esize = dtype_size(dtype);
  if (esize == 0) return DQ_ERR_DTYPE;
  if (T <= 0 || N <= 0 || K <= 0 || ldx < K || ldy < N) return DQ_ERR_INVALID_ARG;
  if (K % 64 != 0) return DQ_ERR_SHAPE;
  if (T > ((int64_t)1 << 30) || N > ((int64_t)1 << 30) || K > ((int64_t)1 << 30))
    return DQ_ERR_SHAPE;
  if (X == nullptr || w_packed == nullptr || w_scales == nullptr || w_tensor_scale == nullptr ||
      y == nullptr)
    return DQ_ERR_INVALID_ARG;
  if (!aligned16(X) || (ldx * esize) % 16 != 0) return DQ_ERR_INVALID_ARG;
  if (c != nullptr && !aligned16(c)) return DQ_ERR_INVALID_ARG;
  if (!aligned16(w_packed) || (reinterpret_cast<uintptr_t>(w_scales) & 3u) ||
      (reinterpret_cast<uintptr_t>(y) & 3u))
    return DQ_ERR_INVALID_ARG;
  const LinearWs l = linear_ws(T, N, K);
  if (workspace == nullptr || workspace_bytes < l.total) return DQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return DQ_ERR_INVALID_ARG;
  unsigned* errp = nullptr;
  if ((st = err_word_ptr(&errp)) != DQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int64_t kq = K / 64;
  // the scale factors of the rows past T in the last 128-row block
  if (T % 128 != 0 &&
      (st = from_cuda(cudaMemsetAsync(ws + l.sfa + (T / 128) * kq * 512, 0, (size_t)kq * 512, s))) != DQ_OK)
    return st;
  // one pass over X: fl32(X * c) quantized, codes and scale factors in the GEMM's layouts
  dq::ActLaunch act = {};
  act.X = X;
  act.tokens = T;
  act.n = K;
  act.ldx = ldx;
  act.c = c;
  act.x_packed = ws + l.codes;
  act.scales = ws + l.sfa;
  act.tensor_scale = reinterpret_cast<float*>(ws);
  act.partials = reinterpret_cast<unsigned*>(ws + 256);
  act.err_word = errp;
  act.sf_tc = 1;
  if ((st = from_cuda(dq::launch_act(act, fmt.kind, fmt.group, esize, s))) != DQ_OK) return st;
  dq::GemmArgs A = {};
  A.xq = ws + l.codes;
  A.xs = nullptr;
  A.xst = reinterpret_cast<const float*>(ws);
  A.wq = w_packed;
  A.ws = w_scales;
  A.wst = w_tensor_scale;
  A.y = y;
  A.T = T;
  A.N = N;
  A.K = K;
  A.ldy = ldy;
  A.err_word = errp;
  A.sfa = ws + l.sfa;
  return from_cuda(dq::launch_w4a4_gemm(A, ws + l.sfb, s));
}

dq_status dq_encode(const float* x, int64_t count, int32_t codec, void* codes, void* stream) {
  if (codec < DQ_CODEC_INT4 || codec > DQ_CODEC_INT8) return DQ_ERR_DTYPE;
  if (count < 0) return DQ_ERR_INVALID_ARG;
  if (count > 0 && (x == nullptr || codes == nullptr)) return DQ_ERR_INVALID_ARG;
  return from_cuda(dq::launch_encode(x, count, codec, codes, static_cast<cudaStream_t>(stream)));
}

dq_status dq_decode(const void* codes, int64_t count, int32_t codec, float* x, void* stream) {
  if (codec < DQ_CODEC_INT4 || codec > DQ_CODEC_INT8) return DQ_ERR_DTYPE;
  if (count < 0) return DQ_ERR_INVALID_ARG;
  if (count > 0 && (x == nullptr || codes == nullptr)) return DQ_ERR_INVALID_ARG;
  return from_cuda(dq::launch_decode(codes, count, codec, x, static_cast<cudaStream_t>(stream)));
}

dq_status dq_set_timing_events(void* const* start_events, void* const* stop_events,
                               int32_t capacity) {
  if (capacity < 0) return DQ_ERR_INVALID_ARG;
  if (capacity > 0 && (start_events == nullptr || stop_events == nullptr)) return DQ_ERR_INVALID_ARG;
  t_ev_start = capacity > 0 ? start_events : nullptr;
  t_ev_stop = capacity > 0 ? stop_events : nullptr;
  t_ev_cap = capacity;
  t_ev_used = 0;
  return DQ_OK;
}

int32_t dq_timing_events_used(void) { return t_ev_used; }

int64_t dq_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

dq_status dq_last_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DQ_ERR_CUDA;
  unsigned* p = nullptr;
  dq_status st = err_word_ptr(&p);
  if (st != DQ_OK) return st;
  unsigned h = 0;
  if (cudaMemcpy(&h, p, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return DQ_ERR_CUDA;
  if (h != 0) {
    const unsigned z = 0;
    if (cudaMemcpy(p, &z, sizeof(z), cudaMemcpyHostToDevice) != cudaSuccess) return DQ_ERR_CUDA;
  }
  if (h & 1u) return DQ_ERR_NONFINITE;
  if (h & 2u) return DQ_ERR_TIMEOUT;
  if (h & 4u) return DQ_ERR_INVALID_ARG;
  return DQ_OK;
}

}  // extern "C"
