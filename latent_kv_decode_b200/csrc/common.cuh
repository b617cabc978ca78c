// Shared device helpers of libmla: element conversions, FP4/E4M3 decoding,
// visibility of a cache row, and the parameter block every decode kernel reads.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "../../include/mla.h"

namespace mla {

constexpr int kCkv = 512;          // latent width (DeepSeek kv_lora_rank)
constexpr int kTile = 64;          // split ranges are cut on multiples of 64 tokens
constexpr int kFp4EntryBytes = 288;

// Everything a decode / combine kernel needs, resolved on the host.
struct DecodeParams {
  int B, H, Q, HQ, Ckv, Dr, D;     // D = Ckv + Dr
  const void* q_lat;
  const void* q_pe;
  const void* kv;
  const void* pe;
  int64_t kv_row, pe_row, kv_batch, pe_batch;
  int Lk;
  const int32_t* seq_lens;
  const int32_t* block_table;
  int max_pages, page_size, num_pages;
  const uint8_t* mask;
  int causal;
  float scale;                     // softmax_scale
  float scale_log2;                // softmax_scale * log2(e)
  const float* sinks;
  int rope_tail;
  float rope_theta;
  int num_splits;
  void* x;
  float* lse;
  int32_t* err;
  float* ws_o;                     // (S, B, HQ, Ckv) normalised partial outputs
  float* ws_lse;                   // (S, B, HQ) partial log-sum-exp (natural log)
};

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa.
// Magnitudes by (exponent, mantissa): 0, 0.5 | 1, 1.5 | 2, 3 | 4, 6.
__device__ __forceinline__ float e2m1_value(uint32_t code) {
  const uint32_t e = (code >> 1) & 3u, m = code & 1u;
  const float mag = (e == 0) ? 0.5f * (float)m : (1.0f + 0.5f * (float)m) * (float)(1u << (e - 1));
  return (code & 8u) ? -mag : mag;
}

// E4M3 ("fn"): bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa;
// exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no infinities.
__device__ __forceinline__ float e4m3_value(uint32_t byte) {
  const uint32_t s = (byte >> 7) & 1u, e = (byte >> 3) & 15u, m = byte & 7u;
  float mag;
  if (e == 15u && m == 7u) {
    mag = __int_as_float(0x7fc00000);
  } else if (e == 0u) {
    mag = (float)m * 0.001953125f;  // m * 2^-9
  } else {
    mag = __int_as_float((int)(((e + 120u) << 23) | (m << 20)));  // (1+m/8) 2^(e-7)
  }
  return s ? -mag : mag;
}

__device__ __forceinline__ void flag_error(const DecodeParams& p, int bit) {
  if (p.err) atomicOr(p.err, bit);
}

// Length of sequence b, clamped to [0, Lk]; a length outside that range is
// flagged as a bad table entry.
__device__ __forceinline__ int seq_len_of(const DecodeParams& p, int b) {
  if (!p.seq_lens) return p.Lk;
  const int L = p.seq_lens[b];
  if (L < 0 || L > p.Lk) {
    flag_error(p, MLA_DEVICE_ERR_BLOCK_TABLE);
    return L < 0 ? 0 : p.Lk;
  }
  return L;
}

// Token range [t0, t1) of split z of a sequence of `len` tokens: whole 64-token
// tiles, ceil(tiles / S) per split.
__device__ __forceinline__ void split_range(int len, int S, int z, int& t0, int& t1) {
  const int tiles = (len + kTile - 1) / kTile;
  const int per = (tiles + S - 1) / S;
  t0 = min(len, z * per * kTile);
  t1 = min(len, (z + 1) * per * kTile);
}

// Pool row of token t of sequence b, or -1 when the block table entry is bad.
__device__ __forceinline__ int64_t cache_row(const DecodeParams& p, int b, int t) {
  if (!p.block_table) return (int64_t)t;
  const int page = p.block_table[(int64_t)b * p.max_pages + t / p.page_size];
  if (page < 0 || page >= p.num_pages) return -1;
  return (int64_t)page * p.page_size + (t % p.page_size);
}

// Is token t visible to query q of sequence b (t < len is checked by callers)?
__device__ __forceinline__ bool visible(const DecodeParams& p, int len, int q, int t) {
  if (p.mask && p.mask[t] == 0) return false;
  if (p.causal && t > len - p.Q + q) return false;
  return true;
}

// Inverse RoPE of one (even, odd) pair at position pos: rotate by -pos*theta^(-2j/tail).
// The angle is formed and reduced in double so positions up to 2^31 keep
// full float accuracy.
__device__ __forceinline__ void inverse_rope_pair(float& a, float& b, int j, int tail, float theta,
                                                  int pos) {
  const double freq = pow((double)theta, -2.0 * (double)j / (double)tail);
  const double ang = -(double)pos * freq;
  double s, c;
  sincos(ang, &s, &c);
  const float fa = a, fb = b;
  a = (float)(fa * c - fb * s);
  b = (float)(fa * s + fb * c);
}

}  // namespace mla
