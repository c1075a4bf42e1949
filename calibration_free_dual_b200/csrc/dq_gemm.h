// dq_gemm.h — launch descriptor of the W4A4 GEMM consumer (host API and kernel).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace dq {

// W4A4 GEMM (NVFP4): y[T, N] = dequant(x)[T, K] dequant(w)[N, K]^T * xst * wst
struct GemmArgs {
  const uint8_t* xq;      // [T, K/2] E2M1 codes (low nibble = even column)
  const uint8_t* xs;      // [T, K/16] E4M3 scale codes (0 = an all-zero block)
  const float* xst;       // [1] activation tensor scale
  const uint8_t* wq;      // [N, K/2]
  const uint8_t* ws;      // [N, K/16]
  const float* wst;       // [1] weight tensor scale
  float* y;               // [T, ldy] fp32
  int64_t T, N, K, ldy;
  unsigned* err_word;
  // interleaved scale factors [rows / 128][K / 64][512 bytes]: sfb is set by the launcher
  // (workspace); sfa too when null on entry, else the activation's are already laid out there
  // (rows past T zero) and xs is not read
  const uint8_t* sfa;
  const uint8_t* sfb;
  int store_tma;          // set by the launcher: y is written by TMA tensor stores
};
// sfa_given: the activation's scale factors come laid out (workspace for the weight's only)
size_t gemm_workspace_bytes(int64_t T, int64_t N, int64_t K, bool sfa_given = false);
cudaError_t launch_w4a4_gemm(const GemmArgs& A, void* workspace, cudaStream_t s);

}  // namespace dq
