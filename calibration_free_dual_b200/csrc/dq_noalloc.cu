// dq_noalloc.cu — the dual-scale solve for callers that cannot allocate device memory.
//
// dq_solve needs a caller-provided workspace. Some callers cannot obtain one: a host
// application (an inference server, a plugin host, an embedded runtime) may own every byte
// of device memory through its own pool allocator and not let a library call cudaMalloc
// behind its back, since that would bypass its accounting and can stall the whole device
// while the driver maps memory. dq_solve_noalloc serves those callers: it takes its scratch
// from a fixed array compiled into this library instead of a workspace argument, and calls
// no allocating routine. The caller still provides the inputs and outputs.
#include <cuda.h>   // CUcontext (the two driver calls below are fetched from the driver)
#include <mutex>

#include "dq.h"
#include "dq_internal.h"

namespace {

// The fixed scratch. Every GPU that loads the library holds these bytes until the process
// exits. Host code must not hand this name to a kernel: on the host it is only a stand-in
// for the symbol, so its device address is looked up below, once per context.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DQ_NOALLOC_SCRATCH_BYTES];

// A device address is valid only in the context it was looked up in, so the cache is keyed
// by the context's id (unique for the life of the process: a context created after a device
// reset, or a second context on the same device, gets a new one).
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct Entry {
  unsigned long long ctx_id;
  void* addr;
};
constexpr int kMaxContexts = 64;
std::mutex g_mu;
Entry g_cache[kMaxContexts] = {};
int g_used = 0;
CtxGetCurrentFn g_get_current = nullptr;
CtxGetIdFn g_get_id = nullptr;
bool g_loaded = false;

bool load_driver_calls() {
  if (!g_loaded) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess)
      g_get_current = reinterpret_cast<CtxGetCurrentFn>(a);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess)
      g_get_id = reinterpret_cast<CtxGetIdFn>(b);
    (void)cudaGetLastError();
    g_loaded = true;
  }
  return g_get_current != nullptr && g_get_id != nullptr;
}

// Device address of the scratch array in the calling thread's current context (looked up
// with cudaGetSymbolAddress on the first call in that context, which also loads the
// array's module and, for a thread with no context yet, binds the device's primary context).
dq_status scratch_address(void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!load_driver_calls()) return DQ_ERR_CUDA;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  void* p = nullptr;
  if (g_get_current(&ctx) != CUDA_SUCCESS) return DQ_ERR_CUDA;
  if (ctx == nullptr) {
    // no context yet: the runtime lookup binds the primary context of the current device
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return DQ_ERR_CUDA;
    }
    if (g_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return DQ_ERR_CUDA;
  }
  if (g_get_id(ctx, &id) != CUDA_SUCCESS) return DQ_ERR_CUDA;
  for (int i = 0; i < g_used; ++i) {
    if (g_cache[i].ctx_id == id) {
      *out = g_cache[i].addr;
      return DQ_OK;
    }
  }
  if (p == nullptr &&
      (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)) {
    (void)cudaGetLastError();
    return DQ_ERR_CUDA;
  }
  // keep the most recent contexts; a context past the table's size is looked up again
  const int slot = g_used < kMaxContexts ? g_used++ : (int)(id % kMaxContexts);
  g_cache[slot] = Entry{id, p};
  *out = p;
  return DQ_OK;
}

}  // namespace

extern "C" dq_status dq_solve_noalloc(const void* W, int32_t dtype, int64_t m, int64_t n,
                                      int64_t ldw, dq_format fmt, int32_t iters,
                                      const float* r0, const float* c0, uint8_t* q_packed,
                                      float* r, float* c, void* block_scales,
                                      float* tensor_scale, double* mse_trace, void* stream) {
  // the size check comes first and needs no device
  const int64_t mm = m, nn = n;
  const size_t need = (m > 0 && n > 0 && iters >= 0)
                          ? dq_solve_workspace_bytes(1, &mm, &nn, fmt, iters) : 0;
  if (need > DQ_NOALLOC_SCRATCH_BYTES) return DQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    const dq_status st = scratch_address(&scratch);
    if (st != DQ_OK) return st;
  }
  // dq_solve validates every argument, clears the words that must start at zero (the NVFP4
  // amax) with a memset on `stream`, and overwrites every other scratch byte it reads.
  return dq_solve(W, dtype, m, n, ldw, fmt, iters, r0, c0, q_packed, r, c, block_scales,
                  tensor_scale, mse_trace, scratch, scratch ? DQ_NOALLOC_SCRATCH_BYTES : 0,
                  stream);
}
