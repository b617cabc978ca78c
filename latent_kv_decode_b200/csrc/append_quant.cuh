// FP4 quantiser of the shared-latent cache append (the openarchlab
// DeepSeek-V4.1-Flash page "4A · Multi-head Latent Attention", §1 on the
// 288-byte entry and §4 on checking the FP4 latent against float32): one
// group of 16 channels gets scale = E4M3(amax / 6) and codes E2M1(x / scale),
// both rounded to nearest-even with saturation; a zero scale gives zero codes.
//
// The two quotients are float32 (correctly rounded), and the conversions are
// CUDA's float -> FP8 / FP4 intrinsics, so the same function runs on the host
// (their software path) and on the GPU (the hardware conversions). Kept in a
// header of its own so a host program can check it against the format
// definitions without a GPU.
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace mla {

// x: the group's 16 channel values. codes: byte k holds channel 2k in its low
// nibble and channel 2k+1 in its high nibble. Returns the E4M3 scale byte.
__host__ __device__ inline uint8_t fp4_quantize_group16(const float (&x)[16], uint8_t (&codes)[8]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  const uint8_t sbyte = (uint8_t)__nv_cvt_float_to_fp8(amax / 6.0f, __NV_SATFINITE, __NV_E4M3);
  const float s = __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)sbyte, __NV_E4M3)));
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint8_t lo = 0, hi = 0;
    if (s > 0.f) {
      lo = (uint8_t)(__nv_cvt_float_to_fp4(x[2 * k] / s, __NV_E2M1, cudaRoundNearest) & 0xF);
      hi = (uint8_t)(__nv_cvt_float_to_fp4(x[2 * k + 1] / s, __NV_E2M1, cudaRoundNearest) & 0xF);
    }
    codes[k] = (uint8_t)(lo | (hi << 4));
  }
  return sbyte;
}

}  // namespace mla
