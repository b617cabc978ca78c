// Tensor-core per-head projections of the absorbed step (bf16, fp32 accumulate):
//
//   mla_absorb_q  blank [1] of the 6547.cn MLA decode question:
//                 q_lat[b,h,q,c] = sum_d q_nope[b,h,q,d] W_UK[h][d][c]
//                 computed transposed, D[c][n] = W_UK[h]^T . q_nope[n]^T:
//                 M = 128 latent columns per CTA (A = W_UK, MN-major),
//                 N = B*Q query rows, K = Dn.
//   mla_up_proj   blank [5]: out[b,h,q,v] = sum_c x[b,h,q,c] W_UV[h][v][c]
//                 D[v][n] = W_UV[h] . x[n]^T: M = Vd = 128 (A = W_UV,
//                 K-major), N = B*Q, K = Ckv = 512.
//
// One CTA per (head, 128-row M tile). K is walked in 64-wide blocks through a
// ring of shared-memory stages filled by TMA (warp 0) and consumed by single-
// thread tcgen05.mma issue (warp 1); D (128 lanes x N fp32 columns) lives in
// TMEM and all four warps write it out. Both ops stream their weight (16.8 MB
// at H=128) once, so they are HBM-bound; N = B*Q <= 256.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kPThreads = 128;
constexpr int kPStages = 4;
constexpr int kMaxN = 256;

struct alignas(64) ProjParams {
  CUtensorMap tm_a;   // weight
  CUtensorMap tm_b;   // query / latent rows (D, Q, H, B)
  void* out;
  int B, H, Q, N;     // N = B*Q rounded up to a multiple of 16
  int nkb;            // 64-wide K blocks
  int a_mn_major;     // absorb: W_UK read M-major; up: W_UV read K-major
  int row0;           // first weight row of the head's slice (0 for W_UK, Dn for W_UV)
  int out_cols;       // columns per output row: 512 (q_lat) or Vd (out)
  int a_bytes, b_bytes;  // per stage
  int32_t* err;
};

__global__ void __launch_bounds__(kPThreads, 1) proj_sm100_kernel(const __grid_constant__ ProjParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb0 = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sb0 - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, mt = blockIdx.y;
  const int stage_bytes = P.a_bytes + P.b_bytes;
  const uint32_t off_bar = kPStages * stage_bytes;
  auto bar = [&](int i) -> uint32_t { return sb0 + off_bar + 8u * (uint32_t)i; };
  // bars: full[4], empty[4], done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + off_bar + 8 * (2 * kPStages + 1));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + off_bar + 8 * (2 * kPStages + 1) + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(bar(s), 1);
      mbar_init(bar(kPStages + s), 1);
    }
    mbar_init(bar(2 * kPStages), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  auto fail = [&]() {
    *abort_flag = 1;
    if (P.err) atomicOr(P.err, MLA_DEVICE_ERR_TIMEOUT);
  };

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    for (int kb = 0; kb < P.nkb; ++kb) {
      const int s = kb % kPStages;
      if (kb >= kPStages && !mbar_wait(bar(kPStages + s), ((kb / kPStages) - 1) & 1)) {
        fail();
        break;
      }
      const uint32_t a_dst = sb0 + s * stage_bytes, b_dst = a_dst + P.a_bytes;
      mbar_arrive_expect_tx(bar(s), P.a_bytes + P.b_bytes);
      if (P.a_mn_major) {
        // W_UK[h] rows d in [64 kb, 64 kb + 64), columns c in this M tile: two 64-wide MN blocks
        tma_load_3d(a_dst, &P.tm_a, bar(s), 128 * mt, P.row0 + 64 * kb, h);
        tma_load_3d(a_dst + 8192, &P.tm_a, bar(s), 128 * mt + 64, P.row0 + 64 * kb, h);
      } else {
        // W_UV[h] rows v (128), columns c in [64 kb, 64 kb + 64)
        tma_load_3d(a_dst, &P.tm_a, bar(s), 64 * kb, P.row0, h);
      }
      // query rows n = (b, q) of head h, K columns [64 kb, 64 kb + 64)
      asm volatile(
          "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
          " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(b_dst),
          "l"(reinterpret_cast<uint64_t>(&P.tm_b)), "r"(bar(s)), "r"(64 * kb), "r"(0), "r"(h), "r"(0)
          : "memory");
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_bf16_f32(128, P.N, P.a_mn_major != 0, false);
    bool ok = true;
    for (int kb = 0; kb < P.nkb && ok; ++kb) {
      const int s = kb % kPStages;
      if (!mbar_wait(bar(s), (kb / kPStages) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t a = sb0 + s * stage_bytes, bb = a + P.a_bytes;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t ad = P.a_mn_major ? smem_desc(a + 2048 * k, 8192, 1024, kSwizzle128B)
                                         : smem_desc(a + 32 * k, 16, 1024, kSwizzle128B);
        mma_bf16_ss(tmem, ad, smem_desc(bb + 32 * k, 16, 1024, kSwizzle128B), idesc,
                    (kb | k) != 0);
      }
      mma_commit(bar(kPStages + s));
    }
    if (ok) mma_commit(bar(2 * kPStages));
    else fail();
  }
  __syncwarp();

  // ------------------------------------------------------------------ epilogue
  bool ok = mbar_wait(bar(2 * kPStages), 0);
  ok = __all_sync(0xffffffffu, ok) != 0;
  tc_fence_after();
  const int m = 32 * warp + lane;                       // TMEM lane = output column within the tile
  const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
  const int rows = P.B * P.Q;
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(P.out);
  const int col = 128 * mt + m;
  if (ok) {
    for (int n0 = 0; n0 < P.N; n0 += 16) {
      uint32_t v[16];
      tmem_ld16(tmem + lane_base + (uint32_t)n0, v);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int n = n0 + i;
        if (n < rows) {
          const int b = n / P.Q, q = n % P.Q;
          out[(((int64_t)b * P.H + h) * P.Q + q) * P.out_cols + col] =
              __float2bfloat16_rn(__uint_as_float(v[i]));
        }
      }
    }
  } else if (threadIdx.x == 0) {
    fail();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 proj_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool proj_encode(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box) {
  auto fn = proj_encode_fn();
  if (!fn) return false;
  cuuint32_t elem[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
            reinterpret_cast<const cuuint64_t*>(dims),
            reinterpret_cast<const cuuint64_t*>(strides_bytes),
            reinterpret_cast<const cuuint32_t*>(box), elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// rows: (K, Q, H, B) view of a (B, H, Q, K) tensor; box 64 x Q x 1 x ceil(N/Q)
bool encode_rows(CUtensorMap* m, const void* base, int B, int H, int Q, int K, int N) {
  uint64_t d[4] = {(uint64_t)K, (uint64_t)Q, (uint64_t)H, (uint64_t)B};
  uint64_t s[3] = {(uint64_t)K * 2, (uint64_t)Q * K * 2, (uint64_t)H * Q * K * 2};
  uint32_t box[4] = {64, (uint32_t)Q, 1, (uint32_t)((N + Q - 1) / Q)};
  return proj_encode(m, base, 4, d, s, box);
}

cudaError_t launch_proj(bool absorb, const void* act, const void* w, void* out, int B, int H, int Q,
                        int Dn, int Vd, int Ckv, cudaStream_t st) {
  ProjParams P;
  memset(&P, 0, sizeof(P));
  const int rows = B * Q;
  P.out = out;
  P.B = B;
  P.H = H;
  P.Q = Q;
  P.N = ((rows + 15) / 16) * 16;           // a multiple of 16, hence of Q in {1, 2, 4}
  const int K = absorb ? Dn : Ckv;
  P.nkb = K / 64;
  P.b_bytes = P.N * 128;
  uint64_t wd[3] = {(uint64_t)Ckv, (uint64_t)(Dn + Vd), (uint64_t)H};
  uint64_t ws[2] = {(uint64_t)Ckv * 2, (uint64_t)(Dn + Vd) * Ckv * 2};
  if (absorb) {
    P.a_mn_major = 1;
    P.row0 = 0;
    P.out_cols = Ckv;
    P.a_bytes = 2 * 8192;                  // 64 K rows x 2 MN blocks of 128 B
    uint32_t box[3] = {64, 64, 1};
    if (!proj_encode(&P.tm_a, w, 3, wd, ws, box)) return cudaErrorInvalidValue;
  } else {
    P.a_mn_major = 0;
    P.row0 = Dn;
    P.out_cols = Vd;
    P.a_bytes = 128 * 128;                 // 128 M rows x 64 K columns
    uint32_t box[3] = {64, 128, 1};
    if (!proj_encode(&P.tm_a, w, 3, wd, ws, box)) return cudaErrorInvalidValue;
  }
  if (!encode_rows(&P.tm_b, act, B, H, Q, K, P.N)) return cudaErrorInvalidValue;
  const int smem = kPStages * (P.a_bytes + P.b_bytes) + 1024 + 1024;
  cudaError_t e = cudaFuncSetAttribute(proj_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(H, absorb ? Ckv / 128 : Vd / 128);
  proj_sm100_kernel<<<grid, kPThreads, smem, st>>>(P);
  return cudaGetLastError();
}

}  // namespace

bool sm100_proj_supported(int B, int H, int Q, int Dn, int Vd, int Ckv) {
  const int rows = B * Q;
  if (rows < 1 || rows > kMaxN || !(Q == 1 || Q == 2 || Q == 4)) return false;
  if (Dn % 64 != 0 || Vd != 128 || Ckv != 512) return false;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return false;
  return major == 10 && proj_encode_fn() != nullptr;
}

cudaError_t launch_absorb_sm100(const void* q_nope, const void* wkv_b, void* q_lat, int B, int H,
                                int Q, int Dn, int Vd, int Ckv, cudaStream_t st) {
  return launch_proj(true, q_nope, wkv_b, q_lat, B, H, Q, Dn, Vd, Ckv, st);
}

cudaError_t launch_up_proj_sm100(const void* x, const void* wkv_b, void* out, int B, int H, int Q,
                                 int Dn, int Vd, int Ckv, cudaStream_t st) {
  return launch_proj(false, x, wkv_b, out, B, H, Q, Dn, Vd, Ckv, st);
}

}  // namespace mla
