// dq_codec.cu — elementwise encode/decode through the exact device codecs the solver and the
// activation kernel use (for bit-exact tests of the formats).
#include <algorithm>

#include "dq_device.cuh"
#include "dq_internal.h"

namespace dq {
namespace {

__global__ void encode_kernel(const float* x, int64_t count, int codec, void* codes) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float v = x[i];
    switch (codec) {
      case 0: reinterpret_cast<uint8_t*>(codes)[i] = (uint8_t)int4_code(int4_round(v)); break;
      case 1: reinterpret_cast<uint8_t*>(codes)[i] = (uint8_t)(e2m1x2_encode(v, 0.0f) & 0xFu); break;
      case 2: {
        // sign-magnitude E4M3 (RNE, saturating); the solver only encodes v >= 0
        const uint32_t mag = e4m3_encode(fabsf(v));
        reinterpret_cast<uint8_t*>(codes)[i] = (uint8_t)(mag | (signbit(v) ? 0x80u : 0u));
        break;
      }
      case 3: reinterpret_cast<uint8_t*>(codes)[i] = (uint8_t)e8m0_encode(v); break;
      case 4: reinterpret_cast<uint16_t*>(codes)[i] = (uint16_t)bf16_rn_bits(v); break;
      case 5: reinterpret_cast<uint8_t*>(codes)[i] = (uint8_t)int8_code(int8_round(v)); break;
      default: break;
    }
  }
}

__global__ void decode_kernel(const void* codes, int64_t count, int codec, float* x) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x) {
    float v = 0.0f;
    switch (codec) {
      case 0: {
        const int c = reinterpret_cast<const uint8_t*>(codes)[i] & 0xF;
        v = (float)(c >= 8 ? c - 16 : c);
        break;
      }
      case 1: v = e2m1x2_decode(reinterpret_cast<const uint8_t*>(codes)[i] & 0xFu).x; break;
      case 2: {
        const uint32_t c = reinterpret_cast<const uint8_t*>(codes)[i];
        const float mag = e4m3_decode(c & 0x7Fu);
        v = (c & 0x80u) ? -mag : mag;
        break;
      }
      case 3: v = e8m0_decode(reinterpret_cast<const uint8_t*>(codes)[i]); break;
      case 4: v = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(codes)[i] << 16); break;
      case 5: v = (float)reinterpret_cast<const int8_t*>(codes)[i]; break;
      default: break;
    }
    x[i] = v;
  }
}

int grid_for(int64_t count) {
  return (int)std::max<int64_t>(1, std::min<int64_t>((count + 255) / 256, 148 * 32));
}

}  // namespace

cudaError_t launch_encode(const float* x, int64_t count, int codec, void* codes, cudaStream_t s) {
  if (count == 0) return cudaSuccess;
  encode_kernel<<<grid_for(count), 256, 0, s>>>(x, count, codec, codes);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_decode(const void* codes, int64_t count, int codec, float* x, cudaStream_t s) {
  if (count == 0) return cudaSuccess;
  decode_kernel<<<grid_for(count), 256, 0, s>>>(codes, count, codec, x);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace dq
