// Generic CUDA-core kernels of libmla: the float32 path (the question's demo
// shape needs full fp32 accuracy, so no reduced-precision tensor-core math),
// and the path for every shape the tensor-core kernels do not take.
//
//   absorb_q_simt   q_lat = q_nope . W_UK[h]                  (blank [1])
//   up_proj_simt    out   = W_UV[h] . x                       (blank [5])
//   decode_simt     scores, scale, mask, online softmax, latent aggregation
//                   (blanks [2]-[4], step 5), FP4 entries, sinks, inverse RoPE
//   combine_warp    log-sum-exp merge of split partials + epilogue, one or
//                   four warps per row (Ckv = 512, 16-byte aligned buffers)
//   combine_simt    the same merge for any other shape
//
// All arithmetic is float32; inputs are float32 or bf16 (converted on load).
#include "common.cuh"
#include "launch.h"

namespace mla {

// ---------------------------------------------------------------------------
// absorb: grid (H, Ckv/128, ceil(M/32)), 128 threads; thread = one latent column c.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) absorb_q_simt(const T* __restrict__ q_nope,
                                                     const T* __restrict__ wkv_b,
                                                     T* __restrict__ q_lat, int B, int H, int Q,
                                                     int Dn, int Vd, int Ckv) {
  constexpr int MT = 32;
  __shared__ float qs[MT][128 + 1];
  const int h = blockIdx.x;
  const int c = blockIdx.y * 128 + threadIdx.x;
  const int M = B * Q;
  const int m0 = blockIdx.z * MT;
  const int mt = min(MT, M - m0);
  for (int i = threadIdx.x; i < mt * Dn; i += blockDim.x) {
    const int m = i / Dn, d = i % Dn;
    const int b = (m0 + m) / Q, q = (m0 + m) % Q;
    qs[m][d] = to_f32(q_nope[(((int64_t)b * H + h) * Q + q) * Dn + d]);
  }
  __syncthreads();
  float acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0.f;
  const T* w = wkv_b + (int64_t)h * (Dn + Vd) * Ckv + c;
  for (int d = 0; d < Dn; ++d) {
    const float wv = to_f32(w[(int64_t)d * Ckv]);
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = fmaf(qs[m][d], wv, acc[m]);
  }
  for (int m = 0; m < mt; ++m) {
    const int b = (m0 + m) / Q, q = (m0 + m) % Q;
    q_lat[(((int64_t)b * H + h) * Q + q) * Ckv + c] = from_f32<T>(acc[m]);
  }
}

// ---------------------------------------------------------------------------
// up-projection: grid (H, ceil(M/16)), 256 threads = 8 warps, warp w takes
// rows v = w, w+8, ...; lanes split the 512-long dot product.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) up_proj_simt(const T* __restrict__ x,
                                                    const T* __restrict__ wkv_b,
                                                    T* __restrict__ out, int B, int H, int Q,
                                                    int Dn, int Vd, int Ckv) {
  constexpr int MT = 16;
  __shared__ float xs[MT][kCkv];
  const int h = blockIdx.x;
  const int M = B * Q;
  const int m0 = blockIdx.y * MT;
  const int mt = min(MT, M - m0);
  for (int i = threadIdx.x; i < mt * Ckv; i += blockDim.x) {
    const int m = i / Ckv, c = i % Ckv;
    const int b = (m0 + m) / Q, q = (m0 + m) % Q;
    xs[m][c] = to_f32(x[(((int64_t)b * H + h) * Q + q) * Ckv + c]);
  }
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int v = warp; v < Vd; v += 8) {
    const T* w = wkv_b + ((int64_t)h * (Dn + Vd) + Dn + v) * Ckv;
    float wr[kCkv / 32];
#pragma unroll
    for (int i = 0; i < kCkv / 32; ++i) wr[i] = to_f32(w[lane + 32 * i]);
    for (int m = 0; m < mt; ++m) {
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < kCkv / 32; ++i) s = fmaf(xs[m][lane + 32 * i], wr[i], s);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) {
        const int b = (m0 + m) / Q, q = (m0 + m) % Q;
        out[(((int64_t)b * H + h) * Q + q) * Vd + v] = from_f32<T>(s);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// decode: grid (ceil(HQ/16), B, S), 256 threads. A CTA owns 16 query rows of
// one sequence and one split range, walks it in 32-token tiles held in shared
// memory as float32, and keeps the 16 x 512 output accumulator in registers
// (thread = row tid/16, columns tid%16 + 16j).
// ---------------------------------------------------------------------------
constexpr int kRB = 16, kTT = 32;

__host__ __device__ constexpr int simt_pitch(int D) { return D + 1; }

template <typename TQ, bool FP4>
__global__ void __launch_bounds__(256) decode_simt(DecodeParams p) {
  extern __shared__ float smem[];
  const int D = p.D, pitch = simt_pitch(D);
  float* qs = smem;                          // [kRB][pitch]
  float* ks = qs + kRB * pitch;              // [kTT][pitch]
  float* ps = ks + kTT * pitch;              // [kRB][kTT]
  float* alpha_s = ps + kRB * kTT;           // [kRB]
  int* tok_ok = (int*)(alpha_s + kRB);       // [kTT]: row loaded and < len

  const int tid = threadIdx.x;
  const int b = blockIdx.y, z = blockIdx.z;
  const int r0 = blockIdx.x * kRB;
  const int nr = min(kRB, p.HQ - r0);
  const int len = seq_len_of(p, b);
  int t_begin, t_end;
  split_range(len, p.num_splits, z, t_begin, t_end);

  // query rows (r = h*Q + q): latent part then rope part
  const TQ* ql = (const TQ*)p.q_lat;
  const TQ* qp = (const TQ*)p.q_pe;
  for (int i = tid; i < kRB * D; i += blockDim.x) {
    const int r = i / D, k = i % D;
    float v = 0.f;
    if (r < nr) {
      const int64_t row = (int64_t)b * p.HQ + r0 + r;
      v = (k < p.Ckv) ? to_f32(ql[row * p.Ckv + k]) : to_f32(qp[row * p.Dr + (k - p.Ckv)]);
    }
    qs[r * pitch + k] = v;
  }

  // per-row online-softmax state, replicated in the 16 threads of a row
  const int my_r = tid / 16, my_c0 = tid % 16;
  float m_run = -INFINITY, l_run = 0.f;
  float acc[kCkv / 16];
#pragma unroll
  for (int j = 0; j < kCkv / 16; ++j) acc[j] = 0.f;

  for (int t0 = t_begin; t0 < t_end; t0 += kTT) {
    __syncthreads();
    // ---- load tile rows as float32
    if (tid < kTT) {
      const int t = t0 + tid;
      int ok = 0;
      if (t < t_end) {
        ok = cache_row(p, b, t) >= 0;
        if (!ok) flag_error(p, MLA_DEVICE_ERR_BLOCK_TABLE);
      }
      tok_ok[tid] = ok;
    }
    __syncthreads();
    if (FP4) {
      // 288-byte entry: 256 code bytes then 32 scale bytes
      for (int i = tid; i < kTT * (kCkv / 2); i += blockDim.x) {
        const int tt = i / (kCkv / 2), byte = i % (kCkv / 2);
        float lo = 0.f, hi = 0.f;
        if (tok_ok[tt]) {
          const int64_t row = cache_row(p, b, t0 + tt);
          const uint8_t* e = (const uint8_t*)p.kv +
                             (p.block_table ? 0 : (int64_t)b * p.kv_batch) + row * p.kv_row;
          const uint32_t code = e[byte];
          const float sc = e4m3_value(e[kCkv / 2 + (2 * byte) / 16]);
          lo = e2m1_value(code & 15u) * sc;
          hi = e2m1_value(code >> 4) * sc;
        }
        ks[tt * pitch + 2 * byte] = lo;
        ks[tt * pitch + 2 * byte + 1] = hi;
      }
    } else {
      const TQ* kvp = (const TQ*)p.kv;
      const TQ* pep = (const TQ*)p.pe;
      for (int i = tid; i < kTT * D; i += blockDim.x) {
        const int tt = i / D, k = i % D;
        float v = 0.f;
        if (tok_ok[tt]) {
          const int64_t row = cache_row(p, b, t0 + tt);
          if (k < p.Ckv) {
            v = to_f32(kvp[(p.block_table ? 0 : (int64_t)b * p.kv_batch) + row * p.kv_row + k]);
          } else {
            v = to_f32(pep[(p.block_table ? 0 : (int64_t)b * p.pe_batch) + row * p.pe_row +
                           (k - p.Ckv)]);
          }
        }
        ks[tt * pitch + k] = v;
      }
    }
    __syncthreads();
    // ---- scores: thread (token tid%32, rows tid/32 and tid/32 + 8)
    {
      const int tt = tid % kTT;
      const int t = t0 + tt;
      for (int rr = tid / kTT; rr < kRB; rr += 256 / kTT) {
        float s = -INFINITY;
        const int q = (r0 + rr) % p.Q;
        if (rr < nr && tok_ok[tt] && visible(p, len, q, t)) {
          float a = 0.f;
          const float* qrow = qs + rr * pitch;
          const float* krow = ks + tt * pitch;
          for (int k = 0; k < D; ++k) a = fmaf(qrow[k], krow[k], a);
          s = a * p.scale;
        }
        ps[rr * kTT + tt] = s;
      }
    }
    __syncthreads();
    // ---- tile max per row: warp w handles rows w and w+8, lane = token
    {
      const int warp = tid / 32, lane = tid % 32;
      for (int rr = warp; rr < kRB; rr += 8) {
        const float s = ps[rr * kTT + lane];
        float mx = s;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) alpha_s[rr] = mx;  // tile max; the 16 threads of the row read it
      }
    }
    __syncthreads();
    {
      const float tmax = alpha_s[my_r];
      const float m_new = fmaxf(m_run, tmax);
      float alpha = 1.f;
      if (m_new != -INFINITY) alpha = (m_run == -INFINITY) ? 0.f : __expf(m_run - m_new);
      float psum = 0.f;
      for (int tt = 0; tt < kTT; ++tt) {
        const float s = ps[my_r * kTT + tt];
        psum += (s == -INFINITY) ? 0.f : __expf(s - m_new);
      }
      l_run = l_run * alpha + psum;
#pragma unroll
      for (int j = 0; j < kCkv / 16; ++j) acc[j] *= alpha;
      // P . V for this thread's 32 columns
      for (int tt = 0; tt < kTT; ++tt) {
        const float s = ps[my_r * kTT + tt];
        const float pv = (s == -INFINITY) ? 0.f : __expf(s - m_new);
        const float* vrow = ks + tt * pitch;
#pragma unroll
        for (int j = 0; j < kCkv / 16; ++j) acc[j] = fmaf(pv, vrow[my_c0 + 16 * j], acc[j]);
      }
      m_run = m_new;
    }
  }
  __syncthreads();

  // ---- epilogue
  const bool row_ok = my_r < nr;
  const int r = r0 + my_r;
  const int h = r / p.Q, q = r % p.Q;
  const int64_t grow = (int64_t)b * p.HQ + r;
  if (p.num_splits > 1) {
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    if (row_ok) {
      float* o = p.ws_o + ((int64_t)z * p.B * p.HQ + grow) * p.Ckv;
#pragma unroll
      for (int j = 0; j < kCkv / 16; ++j) o[my_c0 + 16 * j] = acc[j] * inv;
      if (my_c0 == 0)
        p.ws_lse[(int64_t)z * p.B * p.HQ + grow] = l_run > 0.f ? m_run + logf(l_run) : -INFINITY;
    }
    return;
  }
  // single split: fold in the sink, normalise, inverse RoPE, store
  float mfin = m_run, lfin = l_run, wscale = 1.f;
  if (p.sinks) {
    const float sk = p.sinks[h];
    const float m2 = fmaxf(m_run, sk);
    const float a = (m_run == -INFINITY) ? 0.f : expf(m_run - m2);
    lfin = l_run * a + expf(sk - m2);
    wscale = a;
    mfin = m2;
  }
  const float inv = lfin > 0.f ? wscale / lfin : 0.f;
  float* xs = ks;  // reuse: [kRB][pitch]
#pragma unroll
  for (int j = 0; j < kCkv / 16; ++j) xs[my_r * pitch + my_c0 + 16 * j] = acc[j] * inv;
  __syncthreads();
  if (p.rope_tail > 0) {
    const int half = p.rope_tail / 2;
    for (int i = tid; i < kRB * half; i += blockDim.x) {
      const int rr = i / half, j = i % half;
      if (rr < nr) {
        const int qq = (r0 + rr) % p.Q;
        const int pos = len - p.Q + qq;
        float* px = xs + rr * pitch + p.Ckv - p.rope_tail + 2 * j;
        inverse_rope_pair(px[0], px[1], j, p.rope_tail, p.rope_theta, pos);
      }
    }
    __syncthreads();
  }
  TQ* xo = (TQ*)p.x;
  for (int i = tid; i < kRB * p.Ckv; i += blockDim.x) {
    const int rr = i / p.Ckv, c = i % p.Ckv;
    if (rr < nr) xo[((int64_t)b * p.HQ + r0 + rr) * p.Ckv + c] = from_f32<TQ>(xs[rr * pitch + c]);
  }
  if (p.lse && row_ok && my_c0 == 0) p.lse[grow] = lfin > 0.f ? mfin + logf(lfin) : -INFINITY;
  (void)q;
}

// ---------------------------------------------------------------------------
// combine: one CTA of 128 threads per row (b, r); thread owns 4 columns.
// ---------------------------------------------------------------------------
template <typename TQ>
__global__ void __launch_bounds__(128) combine_simt(DecodeParams p) {
  __shared__ float xs[kCkv];
  __shared__ float wts[1024];
  __shared__ float red[2];
  const int64_t grow = blockIdx.x;  // b * HQ + r
  const int b = (int)(grow / p.HQ), r = (int)(grow % p.HQ);
  const int h = r / p.Q, q = r % p.Q;
  const int S = p.num_splits;
  const int64_t sstride = (int64_t)p.B * p.HQ;
  if (threadIdx.x == 0) {
    float m = p.sinks ? p.sinks[h] : -INFINITY;
    for (int s = 0; s < S; ++s) m = fmaxf(m, p.ws_lse[s * sstride + grow]);
    float den = 0.f;
    if (m != -INFINITY) {
      for (int s = 0; s < S; ++s) {
        const float l = p.ws_lse[s * sstride + grow];
        den += (l == -INFINITY) ? 0.f : expf(l - m);
      }
      if (p.sinks) den += expf(p.sinks[h] - m);
    }
    const float L = den > 0.f ? m + logf(den) : -INFINITY;
    red[0] = L;
    for (int s = 0; s < S; ++s) {
      const float l = p.ws_lse[s * sstride + grow];
      wts[s] = (l == -INFINITY || L == -INFINITY) ? 0.f : expf(l - L);
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < p.Ckv; c += blockDim.x) {
    float a = 0.f;
    for (int s = 0; s < S; ++s) {
      const float w = wts[s];
      if (w != 0.f) a = fmaf(w, p.ws_o[(s * sstride + grow) * p.Ckv + c], a);
    }
    xs[c] = a;
  }
  __syncthreads();
  if (p.rope_tail > 0) {
    const int len = seq_len_of(p, b);
    for (int j = threadIdx.x; j < p.rope_tail / 2; j += blockDim.x) {
      float* px = xs + p.Ckv - p.rope_tail + 2 * j;
      inverse_rope_pair(px[0], px[1], j, p.rope_tail, p.rope_theta, len - p.Q + q);
    }
    __syncthreads();
  }
  TQ* xo = (TQ*)p.x;
  for (int c = threadIdx.x; c < p.Ckv; c += blockDim.x) xo[grow * p.Ckv + c] = from_f32<TQ>(xs[c]);
  if (p.lse && threadIdx.x == 0) p.lse[grow] = red[0];
}

// combine, kParts warps per row, each over Ckv / kParts columns: Ckv =
// 32 * kCols * kParts. Every warp of a row reduces the splits' lse values
// across its lanes (the same few floats); lane i of part k owns columns
// [Ckv k / kParts + kCols i, + kCols) and issues all its 16-byte partial-O
// loads of a group of splits before using them, so a row costs a few memory
// latencies rather than one per split, and several warps per row keep
// enough loads in flight when rows are few.
template <typename TQ, int kCols, int kParts>
__global__ void __launch_bounds__(128) combine_warp(DecodeParams p) {
  constexpr int kSplitGroup = 4;
  const int lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int64_t grow = gw / kParts;                                    // b * HQ + r
  const int part = (int)(gw % kParts);
  if (grow >= (int64_t)p.B * p.HQ) return;                             // whole warp
  const int b = (int)(grow / p.HQ), r = (int)(grow % p.HQ);
  const int h = r / p.Q, q = r % p.Q;
  const int S = p.num_splits;
  const int64_t sstride = (int64_t)p.B * p.HQ;
  float m = p.sinks ? p.sinks[h] : -INFINITY;
  for (int s = lane; s < S; s += 32) m = fmaxf(m, p.ws_lse[s * sstride + grow]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float den = 0.f;
  if (m != -INFINITY) {
    for (int s = lane; s < S; s += 32) {
      const float l = p.ws_lse[s * sstride + grow];
      den += (l == -INFINITY) ? 0.f : expf(l - m);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (p.sinks) den += expf(p.sinks[h] - m);
  }
  const float L = den > 0.f ? m + logf(den) : -INFINITY;

  const int c0 = part * (32 * kCols) + lane * kCols;
  float acc[kCols];
#pragma unroll
  for (int i = 0; i < kCols; ++i) acc[i] = 0.f;
  for (int s0 = 0; s0 < S; s0 += kSplitGroup) {
    float4 v[kSplitGroup][kCols / 4];
    float w[kSplitGroup];
#pragma unroll
    for (int g = 0; g < kSplitGroup; ++g) {
      const int s = min(s0 + g, S - 1);
      const float l = p.ws_lse[s * sstride + grow];
      w[g] = (s0 + g >= S || l == -INFINITY || L == -INFINITY) ? 0.f : expf(l - L);
      const float4* src = reinterpret_cast<const float4*>(p.ws_o + (s * sstride + grow) * p.Ckv + c0);
#pragma unroll
      for (int i = 0; i < kCols / 4; ++i) v[g][i] = src[i];
    }
#pragma unroll
    for (int g = 0; g < kSplitGroup; ++g) {
      if (w[g] == 0.f) continue;
#pragma unroll
      for (int i = 0; i < kCols / 4; ++i) {
        acc[4 * i] = fmaf(w[g], v[g][i].x, acc[4 * i]);
        acc[4 * i + 1] = fmaf(w[g], v[g][i].y, acc[4 * i + 1]);
        acc[4 * i + 2] = fmaf(w[g], v[g][i].z, acc[4 * i + 2]);
        acc[4 * i + 3] = fmaf(w[g], v[g][i].w, acc[4 * i + 3]);
      }
    }
  }
  const int base = p.Ckv - p.rope_tail;
  if (p.rope_tail > 0 && (part + 1) * (32 * kCols) > base) {           // warp-uniform: this part holds tail dims
    const int pos = seq_len_of(p, b) - p.Q + q;
    if (p.rope_tail <= 64) {
      // lane j evaluates pair j's rotation once (the same double-precision
      // angle as inverse_rope_pair); the lanes owning the tail take it by shuffle
      double cj = 1.0, sj = 0.0;
      if (2 * lane < p.rope_tail) {
        const double freq = pow((double)p.rope_theta, -2.0 * (double)lane / (double)p.rope_tail);
        sincos(-(double)pos * freq, &sj, &cj);
      }
#pragma unroll
      for (int i = 0; i < kCols; i += 2) {
        const int c = c0 + i;
        const int jp = c >= base ? (c - base) >> 1 : 0;
        const double cr = __shfl_sync(0xffffffffu, cj, jp), sr = __shfl_sync(0xffffffffu, sj, jp);
        if (c >= base) {
          const float fa = acc[i], fb = acc[i + 1];
          acc[i] = (float)(fa * cr - fb * sr);
          acc[i + 1] = (float)(fa * sr + fb * cr);
        }
      }
    } else if (c0 + kCols > base) {
#pragma unroll
      for (int i = 0; i < kCols; i += 2) {
        const int c = c0 + i;
        if (c >= base) inverse_rope_pair(acc[i], acc[i + 1], (c - base) >> 1, p.rope_tail, p.rope_theta, pos);
      }
    }
  }
  TQ* xo = reinterpret_cast<TQ*>(p.x) + grow * p.Ckv + c0;
  if constexpr (sizeof(TQ) == 2) {
    static_assert(kCols % 4 == 0, "bf16 stores take 4 columns at a time");
#pragma unroll
    for (int i = 0; i < kCols; i += 4) {
      const __nv_bfloat162 t0 = __floats2bfloat162_rn(acc[i], acc[i + 1]);
      const __nv_bfloat162 t1 = __floats2bfloat162_rn(acc[i + 2], acc[i + 3]);
      *reinterpret_cast<uint2*>(xo + i) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&t0), *reinterpret_cast<const uint32_t*>(&t1));
    }
  } else {
#pragma unroll
    for (int i = 0; i < kCols; i += 4)
      *reinterpret_cast<float4*>(xo + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
  }
  if (p.lse && lane == 0 && part == 0) p.lse[grow] = L;
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
template <typename T>
static cudaError_t absorb_launch(const void* qn, const void* w, void* ql, int B, int H, int Q,
                                 int Dn, int Vd, int Ckv, cudaStream_t st) {
  const int M = B * Q;
  dim3 grid(H, Ckv / 128, (M + 31) / 32);
  absorb_q_simt<T><<<grid, 128, 0, st>>>((const T*)qn, (const T*)w, (T*)ql, B, H, Q, Dn, Vd, Ckv);
  return cudaGetLastError();
}

cudaError_t launch_absorb_simt(const void* qn, const void* w, void* ql, int B, int H, int Q,
                               int Dn, int Vd, int Ckv, bool bf16, cudaStream_t st) {
  return bf16 ? absorb_launch<__nv_bfloat16>(qn, w, ql, B, H, Q, Dn, Vd, Ckv, st)
              : absorb_launch<float>(qn, w, ql, B, H, Q, Dn, Vd, Ckv, st);
}

template <typename T>
static cudaError_t up_launch(const void* x, const void* w, void* out, int B, int H, int Q, int Dn,
                             int Vd, int Ckv, cudaStream_t st) {
  const int M = B * Q;
  dim3 grid(H, (M + 15) / 16);
  up_proj_simt<T><<<grid, 256, 0, st>>>((const T*)x, (const T*)w, (T*)out, B, H, Q, Dn, Vd, Ckv);
  return cudaGetLastError();
}

cudaError_t launch_up_proj_simt(const void* x, const void* w, void* out, int B, int H, int Q,
                                int Dn, int Vd, int Ckv, bool bf16, cudaStream_t st) {
  return bf16 ? up_launch<__nv_bfloat16>(x, w, out, B, H, Q, Dn, Vd, Ckv, st)
              : up_launch<float>(x, w, out, B, H, Q, Dn, Vd, Ckv, st);
}

size_t decode_simt_smem(int D) {
  return sizeof(float) * ((size_t)(kRB + kTT) * simt_pitch(D) + kRB * kTT + kRB) +
         sizeof(int) * kTT;
}

template <typename TQ, bool FP4>
static cudaError_t decode_launch(const DecodeParams& p, cudaStream_t st) {
  const size_t smem = decode_simt_smem(p.D);
  auto kern = decode_simt<TQ, FP4>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.HQ + kRB - 1) / kRB, p.B, p.num_splits);
  kern<<<grid, 256, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode_simt(const DecodeParams& p, bool bf16, bool fp4, cudaStream_t st) {
  if (fp4) return decode_launch<__nv_bfloat16, true>(p, st);
  return bf16 ? decode_launch<__nv_bfloat16, false>(p, st) : decode_launch<float, false>(p, st);
}

template <typename TQ, int kParts>
static cudaError_t combine_warp_launch(const DecodeParams& p, cudaStream_t st) {
  const unsigned grid = (unsigned)(((int64_t)p.B * p.HQ * kParts + 3) / 4);
  combine_warp<TQ, kCkv / (32 * kParts), kParts><<<grid, 128, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_combine_simt(const DecodeParams& p, bool bf16, cudaStream_t st) {
  const int64_t rows = (int64_t)p.B * p.HQ;
  // 16-byte partial loads and 8- or 16-byte stores: the partials and outputs
  // are row-contiguous with rows of Ckv elements, and the buffers come from
  // the allocator
  const bool vec = p.Ckv == kCkv &&
                   (reinterpret_cast<uintptr_t>(p.ws_o) & 15u) == 0 &&
                   (reinterpret_cast<uintptr_t>(p.x) & 15u) == 0 && (p.rope_tail & 1) == 0;
  if (vec) {
    // few rows (long contexts, small batches): four warps per row keep enough
    // loads in flight (measured on B200: 512 rows x 18 splits 12.2 -> 10.3
    // us); many rows fill the GPU with one warp each (2048 rows x 4 splits:
    // 12.4 us with one, 13.7 us with four)
    if (rows < 1024)
      return bf16 ? combine_warp_launch<__nv_bfloat16, 4>(p, st) : combine_warp_launch<float, 4>(p, st);
    return bf16 ? combine_warp_launch<__nv_bfloat16, 1>(p, st) : combine_warp_launch<float, 1>(p, st);
  }
  if (bf16)
    combine_simt<__nv_bfloat16><<<(unsigned)rows, 128, 0, st>>>(p);
  else
    combine_simt<float><<<(unsigned)rows, 128, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace mla
