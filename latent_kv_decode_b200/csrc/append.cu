// Cache append, the step before the decode: each sequence's Q new tokens go
// to the cache rows the decode reads (the neuronix DeepSeek-V3/R1 page's
// LatentKVCachePool slot of a token's latent and rope parts; the openarchlab
// DeepSeek-V4.1-Flash page "4A", §1 and §4, for the shared latent stored as a
// 288-byte FP4 entry with its tail rotated at the token's position).
//
//   append_copy<T>  one warp per new token: copies the Ckv latent and Dr rope
//                   elements into the token's rows.
//   append_fp4      one warp per new token, lane i owns channels 16i..16i+15
//                   (exactly one scale group): loads them, rotates the tail
//                   pairs at the token's position, quantises the group
//                   (append_quant.cuh) and writes its 8 code bytes and its
//                   scale byte of the entry.
//
// Tokens whose position or page is out of range set the error bit and are
// skipped; no access leaves the caller's buffers.
#include <cuda_bf16.h>
#include <math.h>

#include "append.h"
#include "append_quant.cuh"
#include "common.cuh"

namespace mla {
namespace {

constexpr int kAppendWarps = 4;   // tokens per CTA

struct AppendParams {
  int B, Q, Ckv, Dr;
  const void* c_kv;
  const void* k_pe;
  void* kv;
  void* pe;
  int64_t kv_row, pe_row, kv_batch, pe_batch;
  int Lk;
  const int32_t* seq_lens;
  const int32_t* block_table;
  int max_pages, page_size, num_pages;
  int rope_tail;
  float rope_theta;
  int32_t* err;
};

// Cache row of token t of sequence b: (slot, batch) such that the row starts
// at batch * batch_stride + slot * row_stride; false (flagged) when t or its
// page is out of range.
__device__ __forceinline__ bool append_slot(const AppendParams& p, int b, int t, int64_t& slot,
                                            int64_t& batch) {
  if (t < 0 || t >= p.Lk) return false;
  if (!p.block_table) {
    slot = t;
    batch = b;
    return true;
  }
  const int page = p.block_table[(int64_t)b * p.max_pages + t / p.page_size];
  if (page < 0 || page >= p.num_pages) return false;
  slot = (int64_t)page * p.page_size + t % p.page_size;
  batch = 0;
  return true;
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__global__ void __launch_bounds__(32 * kAppendWarps) append_copy(const AppendParams p) {
  const int w = blockIdx.x * kAppendWarps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (w >= p.B * p.Q) return;                      // whole warp
  const int b = w / p.Q, i = w - b * p.Q;
  const int t = p.seq_lens[b] - p.Q + i;
  int64_t slot = 0, batch = 0;
  if (!append_slot(p, b, t, slot, batch)) {
    if (lane == 0 && p.err) atomicOr(p.err, MLA_DEVICE_ERR_BLOCK_TABLE);
    return;
  }
  const T* src = reinterpret_cast<const T*>(p.c_kv) + (int64_t)w * p.Ckv;
  T* dst = reinterpret_cast<T*>(p.kv) + batch * p.kv_batch + slot * p.kv_row;
  for (int c = lane; c < p.Ckv; c += 32) dst[c] = src[c];
  if (p.Dr > 0) {
    const T* sp = reinterpret_cast<const T*>(p.k_pe) + (int64_t)w * p.Dr;
    T* dp = reinterpret_cast<T*>(p.pe) + batch * p.pe_batch + slot * p.pe_row;
    for (int c = lane; c < p.Dr; c += 32) dp[c] = sp[c];
  }
}

template <typename T>
__global__ void __launch_bounds__(32 * kAppendWarps) append_fp4(const AppendParams p) {
  const int w = blockIdx.x * kAppendWarps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (w >= p.B * p.Q) return;                      // whole warp
  const int b = w / p.Q, i = w - b * p.Q;
  const int t = p.seq_lens[b] - p.Q + i;
  int64_t slot = 0, batch = 0;
  if (!append_slot(p, b, t, slot, batch)) {
    if (lane == 0 && p.err) atomicOr(p.err, MLA_DEVICE_ERR_BLOCK_TABLE);
    return;
  }
  const T* src = reinterpret_cast<const T*>(p.c_kv) + (int64_t)w * kCkv + 16 * lane;
  float x[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) x[k] = to_f32(src[k]);
  // RoPE on the tail at position t: pair (base + 2j, base + 2j + 1) turns by
  // t * theta^(-2j/tail); the angle and the rotation in double, as in the
  // decode epilogue's inverse rotation
  const int base = kCkv - p.rope_tail;
  if (p.rope_tail > 0 && 16 * lane + 16 > base) {
#pragma unroll
    for (int k = 0; k < 16; k += 2) {
      const int c = 16 * lane + k;
      if (c >= base) {
        const double freq = pow((double)p.rope_theta, -2.0 * (double)((c - base) >> 1) / (double)p.rope_tail);
        double sn, cs;
        sincos((double)t * freq, &sn, &cs);
        const double a = x[k], bb = x[k + 1];
        x[k] = (float)(a * cs - bb * sn);
        x[k + 1] = (float)(a * sn + bb * cs);
      }
    }
  }
  uint8_t codes[8];
  const uint8_t sbyte = fp4_quantize_group16(x, codes);
  uint8_t* e = reinterpret_cast<uint8_t*>(p.kv) + batch * p.kv_batch + slot * p.kv_row;
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    lo |= (uint32_t)codes[k] << (8 * k);
    hi |= (uint32_t)codes[4 + k] << (8 * k);
  }
  // bytes 8 lane .. 8 lane + 7 hold channels 16 lane .. 16 lane + 15; the
  // entry starts on a 16-byte boundary (checked on the host)
  *reinterpret_cast<uint2*>(e + 8 * lane) = make_uint2(lo, hi);
  e[kCkv / 2 + lane] = sbyte;   // after the kCkv / 2 code bytes: the group's scale
}

}  // namespace

cudaError_t launch_cache_append(const mla_append_args* a, cudaStream_t st) {
  AppendParams p;
  p.B = a->B;
  p.Q = a->Q;
  p.Ckv = a->Ckv;
  p.Dr = a->Dr;
  p.c_kv = a->c_kv;
  p.k_pe = a->k_pe;
  p.kv = a->kv_cache;
  p.pe = a->pe_cache;
  p.kv_row = a->kv_row_stride;
  p.pe_row = a->pe_row_stride;
  p.kv_batch = a->kv_batch_stride;
  p.pe_batch = a->pe_batch_stride;
  p.Lk = a->Lk;
  p.seq_lens = a->seq_lens;
  p.block_table = a->block_table;
  p.max_pages = a->max_pages;
  p.page_size = a->page_size;
  p.num_pages = a->num_pages;
  p.rope_tail = a->rope_tail;
  p.rope_theta = a->rope_theta;
  p.err = a->err_flag;
  const int64_t tokens = (int64_t)a->B * a->Q;
  const unsigned grid = (unsigned)((tokens + kAppendWarps - 1) / kAppendWarps);
  const bool bf16 = a->src_dtype == MLA_BF16;
  if (a->cache_dtype == MLA_FP4_E2M1_E4M3x16) {
    if (bf16)
      append_fp4<__nv_bfloat16><<<grid, 32 * kAppendWarps, 0, st>>>(p);
    else
      append_fp4<float><<<grid, 32 * kAppendWarps, 0, st>>>(p);
  } else if (bf16) {
    append_copy<__nv_bfloat16><<<grid, 32 * kAppendWarps, 0, st>>>(p);
  } else {
    append_copy<float><<<grid, 32 * kAppendWarps, 0, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace mla
