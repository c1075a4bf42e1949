// dq_noalloc.cu — the dual-scale solve for callers that cannot allocate device memory.
//
// dq_solve needs a caller-provided workspace. Some callers cannot obtain one: a host
// application (an inference server, a plugin host, an embedded runtime) may own every byte
// of device memory through its own pool allocator and not let a library call cudaMalloc
// behind its back, since that would bypass its accounting and can stall the whole device
// while the driver maps memory. dq_solve_noalloc serves those callers: it takes its scratch
// from a fixed array compiled into this library instead of a workspace argument, and calls
// no allocating routine. The caller still provides the inputs and outputs.
#include <mutex>

#include "dq.h"
#include "dq_internal.h"

namespace {

// The fixed scratch. Every GPU that loads the library holds these bytes until the process
// exits. Host code must not hand this name to a kernel: on the host it is only a stand-in
// for the symbol, so its device address is looked up below, once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_dev[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on first use).
dq_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_dev[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return DQ_ERR_CUDA;
    }
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
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
