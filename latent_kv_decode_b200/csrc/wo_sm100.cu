// Grouped low-rank output projection after the inverse RoPE (openarchlab
// DeepSeek-V4.1-Flash course, 4A "Multi-head Latent Attention · latent K/V
// dùng chung, RoPE nửa sau và W_O nhóm": §2 Luồng "Group-LoRA W_O (8 nhóm ×
// 1024)" back to [B, T, D_model]; §3 W_O nhóm: every group of heads has its
// own small projection, the groups' results side by side).
//
//   z[t, gR + r] = sum_k wo_a[g, r, k] u_g[t, k],  u_g[t] = x[b, gH/G .. +H/G, q, :] head-major
//   y[t, n]      = sum_k wo_b[n, k] z[t, k]                          (optional)
//
// with t = b*Q + q. Both are one weight-streaming GEMM, Y^T = W . X^T: the
// weights are the M = 128 operand (K-major TMA boxes of 128 rows x 64), the
// few tokens are N (K-major boxes of the activations, padded to a multiple
// of 16 with the TMA's zero fill), the accumulator sits in TMEM. The work is
// HBM-bound on the weights (C4: 64 MB per factor), so the K axis is split
// across CTAs until the grid covers the SMs twice over (two CTAs per SM, each
// with its own TMA ring), and a small kernel sums the fp32 partials into the
// bf16 output.
//
// Roles (256 threads): warp 0 TMA producer, warp 1 MMA issuer and TMEM
// owner, warps 4-7 epilogue (TMEM lane quarter = warp % 4). Every wait is
// bounded; a timeout sets MLA_DEVICE_ERR_TIMEOUT and skips the output.
#include <cudaTypedefs.h>
#include <string.h>

#include "common.cuh"
#include "launch.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kWoThreads = 256;
constexpr int kWoM = 128;                 // output features per CTA
constexpr int kWoABytes = kWoM * 128;     // one 64-wide K chunk of 128 weight rows
constexpr int kWoSmemCap = 100 * 1024;    // shared memory for the stage ring (two CTAs per SM)

struct alignas(64) WoParams {
  CUtensorMap tm_w;   // weights as (64, N rows, K/64 chunks, G): box 64 x 128 x 1 x 1
  CUtensorMap tm_x;   // activations as (64, Q, B, cpb chunks, blocks): box 64 x Q x Bt x 1 x 1
  int T;              // tokens B*Q
  int Q, Bt, Tpad;    // sequences per token block, MMA N = Bt*Q (a multiple of 16, <= 256)
  int kchunks;        // 64-wide chunks of the contraction
  int cpb;            // chunks per activation block (one head, or the whole row)
  int heads_per_group;// activation blocks per group (H/G; 1 for the second factor)
  int N;              // output features per group (R or D)
  int ldy;            // output row length (G*R or D)
  int S;              // K splits
  int stages;
  __nv_bfloat16* y;   // bf16 output (S == 1)
  float* part;        // fp32 partials [S][T][ldy] (S > 1)
  int32_t* err;
};

__global__ void __launch_bounds__(kWoThreads, 2) wo_gemm_kernel(const __grid_constant__ WoParams a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb0 = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sb0 - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kWoM, g = blockIdx.y;
  const int nsplit = a.S;
  const int s = (int)blockIdx.z % nsplit, tb = (int)blockIdx.z / nsplit;   // K split, token block
  const int b0 = tb * a.Bt;
  // this split's chunks [c0, c1)
  const int per = (a.kchunks + nsplit - 1) / nsplit;
  const int c0 = min(a.kchunks, s * per), c1 = min(a.kchunks, c0 + per);
  const int nk = c1 - c0;

  const uint32_t b_bytes = (uint32_t)a.Tpad * 128u;
  const uint32_t stage_bytes = kWoABytes + b_bytes;
  const int ST = a.stages;
  const uint32_t off_bar = (uint32_t)ST * stage_bytes;
  // barriers: full[ST], empty[ST], done; then the TMEM address and an abort flag
  auto bar = [&](int i) -> uint32_t { return sb0 + off_bar + 8u * (uint32_t)i; };
  const int B_FULL = 0, B_EMPTY = ST, B_DONE = 2 * ST;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + off_bar + 8 * (2 * ST + 1));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + off_bar + 8 * (2 * ST + 1) + 4);
  const uint32_t tcols = a.Tpad <= 32 ? 32u : a.Tpad <= 64 ? 64u : a.Tpad <= 128 ? 128u : 256u;

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * ST + 1; ++i) mbar_init(bar(i), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&a.tm_w);
      tma_prefetch_desc(&a.tm_x);
      auto x_coords = [&](int kc, int& c3, int& c4) {
        c3 = kc % a.cpb;
        c4 = g * a.heads_per_group + kc / a.cpb;
      };
      // weights are a read-only input and stream in while the previous kernel
      // finishes; the activations are read only after pdl_wait()
      const int pre = min(ST, nk);
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(bar(B_FULL + i), stage_bytes);
        tma_load_4d(sb0 + i * stage_bytes, &a.tm_w, bar(B_FULL + i), 0, n0, c0 + i, g);
      }
      pdl_wait();
      for (int i = 0; i < pre; ++i) {
        int c3, c4;
        x_coords(c0 + i, c3, c4);
        tma_load_5d(sb0 + i * stage_bytes + kWoABytes, &a.tm_x, bar(B_FULL + i), 0, 0, b0, c3, c4);
      }
      bool ok = true;
      for (int i = pre; i < nk && ok; ++i) {
        const int st = i % ST;
        ok = mbar_wait(bar(B_EMPTY + st), ((i / ST) - 1) & 1);
        if (!ok) break;
        int c3, c4;
        x_coords(c0 + i, c3, c4);
        mbar_arrive_expect_tx(bar(B_FULL + st), stage_bytes);
        tma_load_4d(sb0 + st * stage_bytes, &a.tm_w, bar(B_FULL + st), 0, n0, c0 + i, g);
        tma_load_5d(sb0 + st * stage_bytes + kWoABytes, &a.tm_x, bar(B_FULL + st), 0, 0, b0, c3, c4);
        if (*abort_flag) ok = false;
      }
      if (!ok) {
        *abort_flag = 1;
        if (a.err) atomicOr(a.err, MLA_DEVICE_ERR_TIMEOUT);
        // let copies already issued land before this CTA's shared memory goes away
        const uint64_t t0 = global_ns();
        while (global_ns() - t0 < 50000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // D[n][t]: A = weight rows n (K-major), B = activation rows t (K-major)
      const uint32_t idesc = idesc_bf16_f32(kWoM, a.Tpad, false, false);
      bool ok = true;
      for (int i = 0; i < nk && ok; ++i) {
        const int st = i % ST;
        ok = mbar_wait(bar(B_FULL + st), (i / ST) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint64_t ad = smem_desc(sb0 + st * stage_bytes, 16, 1024, kSwizzle128B);
        const uint64_t bd = smem_desc(sb0 + st * stage_bytes + kWoABytes, 16, 1024, kSwizzle128B);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_bf16_ss(tmem, desc_advance(ad, 32u * k), desc_advance(bd, 32u * k), idesc, (i | k) != 0);
        mma_commit(bar(B_EMPTY + st));
        if (*abort_flag) ok = false;
      }
      if (ok) {
        mma_commit(bar(B_DONE));
      } else {
        *abort_flag = 1;
        if (a.err) atomicOr(a.err, MLA_DEVICE_ERR_TIMEOUT);
        mbar_arrive(bar(B_DONE));
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- epilogue
    // the output (or the partial-sum buffer) may still be read by the
    // previous kernel: write only once it has completed
    pdl_wait();
    bool done = mbar_wait(bar(B_DONE), 0) && *abort_flag == 0;
    done = __all_sync(0xffffffffu, done) != 0;
    if (!done && lane == 0 && a.err) atomicOr(a.err, MLA_DEVICE_ERR_TIMEOUT);
    tc_fence_after();
    const int q4 = warp & 3;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const int n = n0 + 32 * q4 + lane;                 // this thread's output feature
    const int col = g * a.N + n;                       // its column in the output row
    const int t0 = b0 * a.Q;
    const int tvalid = min(a.Tpad, a.T - t0);
    if (done && nk > 0) {
      for (int c = 0; c < a.Tpad; c += 16) {
        uint32_t d[16];
        tmem_ld16(tmem + lane_base + (uint32_t)c, d);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (c + i < tvalid) {
            const int64_t t = t0 + c + i;
            if (nsplit == 1)
              a.y[t * a.ldy + col] = __float2bfloat16_rn(__uint_as_float(d[i]));
            else
              a.part[((int64_t)s * a.T + t) * a.ldy + col] = __uint_as_float(d[i]);
          }
        }
      }
    } else if (done && nsplit > 1) {
      // an empty split still owns its slice of the partial sums
      for (int c = 0; c < tvalid; ++c) a.part[((int64_t)s * a.T + t0 + c) * a.ldy + col] = 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

// y[t, c] = bf16(sum_s part[s, t, c]), four columns per thread
__global__ void __launch_bounds__(256) wo_reduce_kernel(const float* __restrict__ part,
                                                        __nv_bfloat16* __restrict__ y, int S,
                                                        int64_t count4) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= count4) return;
  float4 acc = reinterpret_cast<const float4*>(part)[i];
  for (int s = 1; s < S; ++s) {
    const float4 v = reinterpret_cast<const float4*>(part)[(int64_t)s * count4 + i];
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
  __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
  reinterpret_cast<__nv_bfloat162*>(y)[2 * i] = lo;
  reinterpret_cast<__nv_bfloat162*>(y)[2 * i + 1] = hi;
}

PFN_cuTensorMapEncodeTiled_v12000 wo_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool wo_encode(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
               const uint32_t* box) {
  auto fn = wo_encode_fn();
  if (!fn) return false;
  cuuint32_t elem[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
            reinterpret_cast<const cuuint64_t*>(dims), reinterpret_cast<const cuuint64_t*>(strides),
            reinterpret_cast<const cuuint32_t*>(box), elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int gcd_int(int a, int b) {
  while (b) {
    const int t = a % b;
    a = b;
    b = t;
  }
  return a;
}

}  // namespace

// Token blocking shared by the launcher and the workspace query: Bt sequences
// per block with Bt*Q a multiple of 16 and at most 256 (the MMA's N).
void wo_token_blocks(int B, int Q, int& Bt, int& nblocks) {
  const int unit = 16 / gcd_int(16, Q);                 // sequences per 16-row step
  int cap = 256 / (unit * Q);
  if (cap < 1) cap = 1;
  const int need = (B + unit - 1) / unit;
  Bt = unit * (need < cap ? need : cap);
  nblocks = (B + Bt - 1) / Bt;
}

// K splits: enough CTAs for two per SM (measured on B200 at the V4.1 shape:
// one CTA per SM with a 200 KB ring, 45.9 us per call; two with 100 KB
// rings and twice the splits, 39.9 us)
int wo_splits(int tiles, int kchunks, int sms) {
  int S = 2 * sms / (tiles > 0 ? tiles : 1);
  if (S < 1) S = 1;
  if (S > kchunks) S = kchunks;
  if (S > 16) S = 16;
  return S;
}

// One weight-streaming GEMM pass. Activation view (64, Q, B, cpb, blocks)
// with byte strides xs[0..3] for dims 1..4; weights (G, N, K) row-major.
cudaError_t wo_pass(const void* act, const uint64_t* xdims, const uint64_t* xs, int cpb, int heads_per_group,
                    const void* w, int G, int N, int K, int B, int Q, int ldy, void* y, float* part, int S,
                    int32_t* err, int sms, cudaStream_t st) {
  WoParams P;
  memset(&P, 0, sizeof(P));
  int Bt, nb;
  wo_token_blocks(B, Q, Bt, nb);
  P.T = B * Q;
  P.Q = Q;
  P.Bt = Bt;
  P.Tpad = Bt * Q;
  P.kchunks = K / 64;
  P.cpb = cpb;
  P.heads_per_group = heads_per_group;
  P.N = N;
  P.ldy = ldy;
  P.S = S;
  P.y = reinterpret_cast<__nv_bfloat16*>(y);
  P.part = part;
  P.err = err;
  const uint32_t stage_bytes = kWoABytes + (uint32_t)P.Tpad * 128u;
  P.stages = (int)(kWoSmemCap / stage_bytes);
  if (P.stages > 8) P.stages = 8;
  if (P.stages < 2) return cudaErrorInvalidValue;
  {
    const uint64_t d[4] = {64, (uint64_t)N, (uint64_t)K / 64, (uint64_t)G};
    const uint64_t s[3] = {(uint64_t)K * 2, 128, (uint64_t)N * K * 2};
    const uint32_t box[4] = {64, (uint32_t)kWoM, 1, 1};
    if (!wo_encode(&P.tm_w, w, 4, d, s, box)) return cudaErrorInvalidValue;
  }
  {
    const uint32_t box[5] = {64, (uint32_t)Q, (uint32_t)Bt, 1, 1};
    if (!wo_encode(&P.tm_x, act, 5, xdims, xs, box)) return cudaErrorInvalidValue;
  }
  const size_t smem = (size_t)P.stages * stage_bytes + 8 * (2 * P.stages + 1) + 8 + 1024;
  cudaError_t e = cudaFuncSetAttribute(wo_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(N / kWoM, G, S * nb);
  cfg.blockDim = dim3(kWoThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, wo_gemm_kernel, P);
  if (e != cudaSuccess || S == 1) return e;
  const int64_t count4 = (int64_t)P.T * ldy / 4;
  cudaLaunchConfig_t rc;
  memset(&rc, 0, sizeof(rc));
  rc.gridDim = dim3((unsigned)((count4 + 255) / 256), 1, 1);
  rc.blockDim = dim3(256, 1, 1);
  rc.stream = st;
  rc.attrs = attr;
  rc.numAttrs = 1;
  return cudaLaunchKernelEx(&rc, wo_reduce_kernel, (const float*)part, reinterpret_cast<__nv_bfloat16*>(y), S,
                            count4);
}

size_t group_wo_workspace_bytes(const mla_group_wo_args* a, int sms) {
  const int T = a->B * a->Q;
  const int K1 = (a->H / a->G) * a->Ckv;
  const int S1 = wo_splits(a->G * a->R / kWoM, K1 / 64, sms);
  size_t bytes = 0;
  if (a->wo_b) bytes += (size_t)T * a->G * a->R * 2;               // z (bf16)
  bytes = (bytes + 255) & ~(size_t)255;
  size_t part = S1 > 1 ? (size_t)S1 * T * a->G * a->R * 4 : 0;
  if (a->wo_b) {
    const int S2 = wo_splits(a->D / kWoM, a->G * a->R / 64, sms);
    const size_t p2 = S2 > 1 ? (size_t)S2 * T * a->D * 4 : 0;
    if (p2 > part) part = p2;
  }
  return bytes + part;
}

cudaError_t launch_group_wo_sm100(const mla_group_wo_args* a, void* ws, int sms, cudaStream_t st) {
  const int B = a->B, H = a->H, Q = a->Q, C = a->Ckv, G = a->G, R = a->R;
  const int T = B * Q, K1 = (H / G) * C, GR = G * R;
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  size_t zbytes = a->wo_b ? (size_t)T * GR * 2 : 0;
  zbytes = (zbytes + 255) & ~(size_t)255;
  void* z = a->wo_b ? (void*)base : a->out;
  float* part = reinterpret_cast<float*>(base + zbytes);
  // pass 1: x (B,H,Q,C) viewed as (64, Q, B, C/64, H); group g reads heads g*H/G ..
  {
    const uint64_t d[5] = {64, (uint64_t)Q, (uint64_t)B, (uint64_t)C / 64, (uint64_t)H};
    const uint64_t s[4] = {(uint64_t)C * 2, (uint64_t)H * Q * C * 2, 128, (uint64_t)Q * C * 2};
    const int S1 = wo_splits(GR / kWoM, K1 / 64, sms);
    cudaError_t e = wo_pass(a->x, d, s, C / 64, H / G, a->wo_a, G, R, K1, B, Q, GR, z, part, S1,
                            a->err_flag, sms, st);
    if (e != cudaSuccess || !a->wo_b) return e;
  }
  // pass 2: z (T, G*R) viewed as (64, Q, B, G*R/64, 1)
  {
    const uint64_t d[5] = {64, (uint64_t)Q, (uint64_t)B, (uint64_t)GR / 64, 1};
    const uint64_t s[4] = {(uint64_t)GR * 2, (uint64_t)Q * GR * 2, 128, (uint64_t)T * GR * 2};
    const int S2 = wo_splits(a->D / kWoM, GR / 64, sms);
    return wo_pass(z, d, s, GR / 64, 1, a->wo_b, 1, a->D, GR, B, Q, a->D, a->out, part, S2, a->err_flag, sms,
                   st);
  }
}

}  // namespace mla
