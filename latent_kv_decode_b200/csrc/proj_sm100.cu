// Tensor-core per-head projections of the absorbed step (bf16, fp32 accumulate):
//
//   mla_absorb_q  blank [1] of the 6547.cn MLA decode question:
//                 q_lat[b,h,q,c] = sum_d q_nope[b,h,q,d] W_UK[h][d][c]
//                 computed transposed, D[c][n] = W_UK[h]^T . q_nope[n]^T:
//                 4 M tiles of 128 latent columns (A = W_UK, MN-major),
//                 N = query rows n = (b, q), K = Dn.
//   mla_up_proj   blank [5]: out[b,h,q,v] = sum_c x[b,h,q,c] W_UV[h][v][c]
//                 D[v][n] = W_UV[h] . x[n]^T: M = Vd = 128 (A = W_UV,
//                 K-major), N = query rows, K = Ckv = 512.
//
// Two kernels. proj_tma_kernel (Q in {1, 2, 4}): one CTA per (head, 64
// query rows); the whole 128 KB weight slice of the head comes in as eight
// 16 KB TMA boxes (one 64-column chunk each, already 128-byte-swizzled),
// issued before the programmatic-launch wait since the weights do not depend
// on the previous kernel, and the MMAs of a chunk are issued as soon as it
// lands; the activation rows of the head come in as one TMA box through a
// (64, Q, B, chunk, H) view. proj_sm100_kernel (any Q) is the earlier design:
//
// One CTA per (head, block of up to 64 query rows); absorb also splits the
// 512 latent columns into two CTAs (two CTAs per SM, all SMs busy). Both ops
// stream a 128 KB weight slice per head (16.8 MB at H = 128) and are
// HBM-bound, so the CTA issues every 16-byte load of its slice and of its
// activation rows at once (512 threads; a warp reads 512 contiguous bytes of a
// weight row; at most 192 KB in flight), stores them into the 128-byte-
// swizzled layouts the MMAs read, and one thread then issues the tcgen05 MMAs
// (K = 16 each) into TMEM. 16 warps move D through shared memory, transposed
// to query rows, and write whole output rows with 16-byte stores. Plain loads
// rather than TMA boxes: a box of 64 columns reads 128 B of every 1 KB weight
// row, eight passes over the same DRAM rows per head.
#include <cudaTypedefs.h>
#include <string.h>

#include "common.cuh"
#include "launch.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kPThreads = 512;
constexpr int kRowsPerCta = 64;    // query rows (MMA N) per CTA
constexpr int kWUnits = 64;        // 16-byte units per weight row (Ckv = 512)
// 16-byte loads per thread: absorb (128 rows x 512 B + 64 rows x 256 B) / 512,
// up (128 + 64 rows x 1 KB) / 512
template <bool kAbsorb>
constexpr int kPieces = kAbsorb ? 10 : 24;

struct ProjArgs {
  const __nv_bfloat16* act;   // q_nope (B,H,Q,Dn) or x (B,H,Q,Ckv)
  const __nv_bfloat16* w;     // wkv_b (H, Dn+Vd, Ckv)
  __nv_bfloat16* out;         // q_lat (B,H,Q,Ckv) or out (B,H,Q,Vd)
  int H, Q, rows;             // rows = B*Q
  int w_head_rows;            // Dn + Vd
  int w_row0;                 // first row of the head's slice: 0 (W_UK) or Dn (W_UV)
  int w_rows;                 // rows of the slice: Dn or Vd
  int K;                      // reduction length: Dn (absorb) or Ckv (up)
  int out_cols;               // Ckv (absorb) or Vd (up)
  int w_units;                // 16-byte units of each weight row loaded per CTA: 32 (absorb) or 64
  int absorb;
  int32_t* err;
};

// Element offset of query row n = b*Q + q of head h in a (B, H, Q, cols) tensor.
__device__ __forceinline__ int64_t row_off(int n, int h, int H, int Q, int cols) {
  const int b = n / Q, q = n - b * Q;
  return (((int64_t)b * H + h) * Q + q) * cols;
}

// Byte offset of 16-byte unit u of row r in a stack of 128-byte-swizzled
// blocks: block u/8 holds units [8(u/8), 8(u/8)+8) of every row.
__device__ __forceinline__ uint32_t sw128_off(int r, int u, uint32_t block_bytes) {
  return (uint32_t)(u >> 3) * block_bytes + (uint32_t)r * 128u +
         ((uint32_t)((u & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <bool kAbsorb>
__global__ void __launch_bounds__(kPThreads, kAbsorb ? 2 : 1) proj_sm100_kernel(const ProjArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb0 = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sb0 - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x;
  const int col_half = blockIdx.y;                // absorb: latent columns [256 col_half, +256)
  const int n0 = blockIdx.z * kRowsPerCta;
  const int nrows = min(kRowsPerCta, a.rows - n0);
  const int N = (nrows + 15) & ~15;               // MMA N: a multiple of 16

  // shared layout: weight slice (w_units/8 blocks of 64 columns x w_rows) |
  // activation rows (K/64 blocks x N rows) | done barrier, TMEM slot. After the
  // MMAs the weight area holds the transposed output rows.
  const int w_units = a.w_units;
  const int w_ushift = 31 - __clz(w_units);
  const uint32_t w_block = (uint32_t)a.w_rows * 128u;
  const uint32_t off_x = (uint32_t)(w_units >> 3) * w_block;
  const int a_units = a.K >> 3;                   // 16-byte units per activation row
  const uint32_t x_block = (uint32_t)N * 128u;
  const uint32_t off_bar = off_x + (uint32_t)(a_units >> 3) * x_block;
  const uint32_t bar_done = sb0 + off_bar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + off_bar + 8);
  const int m_tiles = kAbsorb ? 2 : 1;           // absorb: 256 latent columns = 2 M tiles
  const uint32_t tmem_cols = kAbsorb ? 128u : 64u;  // m_tiles x N (<= 64)

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    mbar_init(bar_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }

  // ---------------------------------------------------------------- loads
  // piece p < nw: unit p % w_units of weight row p / w_units; then unit
  // q % a_units of activation row q / a_units (q = p - nw). All issued before
  // any store.
  const int nw = a.w_rows * w_units;
  const int np = nw + nrows * a_units;
  const int a_shift = 31 - __clz(a_units);        // a_units is a power of two
  const char* wslice = reinterpret_cast<const char*>(
      a.w + ((int64_t)h * a.w_head_rows + a.w_row0) * (kWUnits * 8) + col_half * (w_units * 8));
  // the weight slice is a read-only input: it streams in while the previous
  // kernel finishes; the activation rows are read only after pdl_wait()
  uint4 v[kPieces<kAbsorb>];
  bool waited = false;
#pragma unroll
  for (int i = 0; i < kPieces<kAbsorb>; ++i) {
    const int p = (int)threadIdx.x + i * kPThreads;
    if (p >= nw && !waited) {   // the same i for every thread: nw is a multiple of 512
      pdl_wait();
      waited = true;
    }
    if (p < nw) {
      const int r = p >> w_ushift, u = p & (w_units - 1);
      v[i] = ld_stream(wslice + (int64_t)r * (kWUnits * 16) + u * 16);
    } else if (p < np) {
      const int q = p - nw, r = q >> a_shift, u = q & (a_units - 1);
      v[i] = ld_stream(a.act + row_off(n0 + r, h, a.H, a.Q, a.K) + u * 8);
    }
  }
#pragma unroll
  for (int i = 0; i < kPieces<kAbsorb>; ++i) {
    const int p = (int)threadIdx.x + i * kPThreads;
    if (p < nw) {
      const int r = p >> w_ushift, u = p & (w_units - 1);
      *reinterpret_cast<uint4*>(smem + sw128_off(r, u, w_block)) = v[i];
    } else if (p < np) {
      const int q = p - nw, r = q >> a_shift, u = q & (a_units - 1);
      *reinterpret_cast<uint4*>(smem + off_x + sw128_off(r, u, x_block)) = v[i];
    }
  }
  if (!waited) pdl_wait();
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  // ---------------------------------------------------------------- MMAs
  // lane 0 of warp 0 issues; the warp reconverges before anyone waits on D
  if (threadIdx.x == 0) {
    const int ksteps = a.K >> 4;
    if (kAbsorb) {
      // D[c][n], M tile mt = latent columns [128 mt, 128 mt + 128) of this
      // CTA's half: A = two 64-column blocks of W_UK (MN-major, rows d),
      // B = q_nope rows (K-major)
      const uint32_t idesc = idesc_bf16_f32(128, N, true, false);
      for (int mt = 0; mt < m_tiles; ++mt)
        for (int ks = 0; ks < ksteps; ++ks)
          mma_bf16_ss(tmem + (uint32_t)(mt * N),
                      smem_desc(sb0 + 2u * mt * w_block + 2048u * ks, w_block, 1024, kSwizzle128B),
                      smem_desc(sb0 + off_x + (ks >> 2) * x_block + 32u * (ks & 3), 16, 1024,
                                kSwizzle128B),
                      idesc, ks > 0);
    } else {
      // D[v][n]: A = W_UV rows v (K-major), B = x rows (K-major)
      const uint32_t idesc = idesc_bf16_f32(128, N, false, false);
      for (int ks = 0; ks < ksteps; ++ks)
        mma_bf16_ss(tmem,
                    smem_desc(sb0 + (ks >> 2) * w_block + 32u * (ks & 3), 16, 1024, kSwizzle128B),
                    smem_desc(sb0 + off_x + (ks >> 2) * x_block + 32u * (ks & 3), 16, 1024,
                              kSwizzle128B),
                    idesc, ks > 0);
    }
    mma_commit(bar_done);
  }
  __syncwarp();

  // ---------------------------------------------------------------- epilogue
  // D row m (TMEM lane 32*quadrant + lane of M tile mt) is output column
  // 128 mt + m of the CTA's columns; D column n is query row n. Warp
  // 4 * part + quadrant moves its lanes' columns [c_lo, c_hi) into rows n of
  // a bf16 staging tile (row pitch = the CTA's output columns), then the CTA
  // writes whole rows.
  bool ok = mbar_wait(bar_done, 0);
  ok = __all_sync(0xffffffffu, ok) != 0;
  tc_fence_after();
  const int g = warp & 3, part = warp >> 2;
  const uint32_t lane_base = (uint32_t)(32 * g) << 16;
  const int ocols = 128 * m_tiles;                // output columns of this CTA
  __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(smem);
  if (ok) {
    int mt, c_lo, c_hi;
    if (kAbsorb) {                               // 2 M tiles x 2 column halves of N
      mt = part & 1;
      const int hn = ((N >> 1) + 15) & ~15;
      c_lo = min((part >> 1) * hn, N);
      c_hi = (part >> 1) ? N : min(hn, N);
    } else {                                      // 1 M tile x 4 column quarters of N
      mt = 0;
      c_lo = min(part * 16, N);
      c_hi = min(c_lo + 16, N);
    }
    const int m = 128 * mt + 32 * g + lane;
    for (int c = c_lo; c < c_hi; c += 16) {
      uint32_t d[16];
      tmem_ld16(tmem + lane_base + (uint32_t)(mt * N + c), d);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) stage[(c + i) * ocols + m] = __float2bfloat16_rn(__uint_as_float(d[i]));
    }
  } else if (threadIdx.x == 0 && a.err) {
    atomicOr(a.err, MLA_DEVICE_ERR_TIMEOUT);
  }
  __syncthreads();
  if (ok) {
    const int upr = ocols >> 3;                   // 16-byte units per staged row
    const int col0 = kAbsorb ? 256 * col_half : 0;
    for (int e = threadIdx.x; e < nrows * upr; e += kPThreads) {
      const int n = e / upr, u = e - n * upr;
      *reinterpret_cast<uint4*>(a.out + row_off(n0 + n, h, a.H, a.Q, a.out_cols) + col0 + u * 8) =
          *reinterpret_cast<const uint4*>(stage + n * ocols + u * 8);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}


// ---------------------------------------------------------------------------
// TMA-fed projection
// ---------------------------------------------------------------------------
constexpr int kTThreads = 256;
constexpr int kTRows = 64;          // query rows per CTA (MMA N)

struct alignas(64) ProjTmaArgs {
  CUtensorMap tm_w;   // wkv_b as (64, H*(Dn+Vd) rows, 8 chunks): box 64 x w_rows x 1
  CUtensorMap tm_a;   // activation as (64, Q, B, chunks, H): box 64 x Q x 64/Q x chunks x 1
  __nv_bfloat16* out; // q_lat (B,H,Q,Ckv) or out (B,H,Q,Vd)
  int H, Q, rows, Dn, Vd;
  int w_row0;         // 0 (W_UK) or Dn (W_UV)
  int w_rows;         // Dn or Vd
  int a_chunks;       // 64-column chunks of an activation row: Dn/64 or 8
  int out_cols;       // Ckv or Vd
};

// The absorb splits a head's 512 latent columns over two CTAs (blockIdx.z):
// each loads half of the head's W_UK slice (4 chunks), so two CTAs fit on an
// SM and all SMs get work.
template <bool kAbsorb>
__global__ void __launch_bounds__(kTThreads, 2) proj_tma_kernel(const __grid_constant__ ProjTmaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb0 = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sb0 - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x;
  const int bq = kTRows / a.Q;                    // sequences per CTA
  const int n0 = blockIdx.y * kTRows;
  const int nrows = min(kTRows, a.rows - n0);
  constexpr int kWChunks = kAbsorb ? 4 : 8;       // weight chunks of 64 columns in this CTA
  const int hz = kAbsorb ? (int)blockIdx.z : 0;   // absorb: latent columns [256 hz, 256 hz + 256)

  // shared layout: weight chunks (kWChunks x w_rows x 128 B) | activation chunks
  // (a_chunks x 64 rows x 128 B) | barriers: 8 weight chunks, activations, MMAs done
  const uint32_t w_block = (uint32_t)a.w_rows * 128u;
  const uint32_t off_a = (uint32_t)kWChunks * w_block;
  const uint32_t off_bar = off_a + (uint32_t)a.a_chunks * (kTRows * 128u);
  auto bar = [&](int i) -> uint32_t { return sb0 + off_bar + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + off_bar + 8 * 10);
  constexpr uint32_t kTmemCols = kAbsorb ? 128u : 64u;

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < 10; ++i) mbar_init(bar(i), 1);
    *reinterpret_cast<volatile int*>(smem + off_bar + 96) = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  bool ok = true;
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&a.tm_w);
      tma_prefetch_desc(&a.tm_a);
      // the weights are a read-only input: they stream in while the previous
      // kernel finishes; the activations are read only after pdl_wait()
      const int wrow = h * (a.Dn + a.Vd) + a.w_row0;
      for (int j = 0; j < kWChunks; ++j) {
        mbar_arrive_expect_tx(bar(j), w_block);
        tma_load_3d(sb0 + j * w_block, &a.tm_w, bar(j), 0, wrow, 4 * hz + j);
      }
      pdl_wait();
      mbar_arrive_expect_tx(bar(8), (uint32_t)a.a_chunks * kTRows * 128u);
      tma_load_5d(sb0 + off_a, &a.tm_a, bar(8), 0, 0, blockIdx.y * bq, 0, h);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      ok = mbar_wait(bar(8), 0);
      if (kAbsorb) {
        // D[c][n], this CTA's M tile mt = latent columns [256 hz + 128 mt, +128)
        // = its weight chunks 2 mt, 2 mt + 1: A = W_UK^T (MN-major, K = the Dn
        // rows d), B = q_nope rows (K-major)
        const uint32_t idesc = idesc_bf16_f32(128, kTRows, true, false);
        const int ksteps = a.Dn >> 4;
        for (int mt = 0; mt < 2 && ok; ++mt) {
          ok = mbar_wait(bar(2 * mt), 0) && mbar_wait(bar(2 * mt + 1), 0);
          if (!ok) break;
          tc_fence_after();
          const uint64_t ad = smem_desc(sb0 + 2u * mt * w_block, w_block, 1024, kSwizzle128B);
          const uint64_t bd = smem_desc(sb0 + off_a, 16, 1024, kSwizzle128B);
          for (int ks = 0; ks < ksteps; ++ks)
            mma_bf16_ss(tmem + (uint32_t)(mt * kTRows), desc_advance(ad, 2048u * ks),
                        desc_advance(bd, (ks >> 2) * (kTRows * 128u) + 32u * (ks & 3)), idesc, ks > 0);
        }
      } else {
        // D[v][n]: A = W_UV rows v (K-major chunk j), B = x rows (K-major chunk j)
        const uint32_t idesc = idesc_bf16_f32(128, kTRows, false, false);
        for (int j = 0; j < 8 && ok; ++j) {
          ok = mbar_wait(bar(j), 0);
          if (!ok) break;
          tc_fence_after();
          const uint64_t ad = smem_desc(sb0 + j * w_block, 16, 1024, kSwizzle128B);
          const uint64_t bd = smem_desc(sb0 + off_a + j * (kTRows * 128u), 16, 1024, kSwizzle128B);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16_ss(tmem, desc_advance(ad, 32u * k), desc_advance(bd, 32u * k), idesc, (j | k) != 0);
        }
      }
      if (ok) {
        mma_commit(bar(9));
      } else {
        // unblock the epilogue; nothing is written
        *reinterpret_cast<volatile int*>(smem + off_bar + 96) = 1;
        mbar_arrive(bar(9));
        const uint64_t t0 = global_ns();
        while (global_ns() - t0 < 50000ull) {
        }
      }
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- epilogue
  // all 8 warps: TMEM lane quarter g = warp % 4, column half part = warp / 4
  bool done = mbar_wait(bar(9), 0) && *reinterpret_cast<volatile int*>(smem + off_bar + 96) == 0;
  done = __all_sync(0xffffffffu, done) != 0;
  tc_fence_after();
  const int g = warp & 3, part = warp >> 2;
  const uint32_t lane_base = (uint32_t)(32 * g) << 16;
  __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(smem);   // weight area, free now
  const int ocols = kAbsorb ? 256 : 128;            // this CTA's output columns
  if (done) {
    {
      const int mt = kAbsorb ? part : 0;
      const int m = 128 * mt + 32 * g + lane;     // this CTA's output column
      const int c0 = kAbsorb ? 0 : 32 * part;     // absorb: a warp takes all 64 rows of its tiles
      const int c1 = kAbsorb ? kTRows : c0 + 32;
      for (int c = c0; c < c1; c += 16) {
        uint32_t d[16];
        tmem_ld16(tmem + lane_base + (uint32_t)(mt * kTRows + c), d);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) stage[(c + i) * ocols + m] = __float2bfloat16_rn(__uint_as_float(d[i]));
      }
    }
  }
  __syncthreads();
  if (done) {
    const int upr = ocols >> 3;                   // 16-byte units per output row
    for (int e = threadIdx.x; e < nrows * upr; e += kTThreads) {
      const int n = e / upr, u = e - n * upr;
      *reinterpret_cast<uint4*>(a.out + row_off(n0 + n, h, a.H, a.Q, a.out_cols) + ocols * hz + u * 8) =
          *reinterpret_cast<const uint4*>(stage + n * ocols + u * 8);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 proj_encode_fn() {
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

bool proj_encode(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
                 const uint32_t* box) {
  auto fn = proj_encode_fn();
  if (!fn) return false;
  cuuint32_t elem[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
            reinterpret_cast<const cuuint64_t*>(dims), reinterpret_cast<const cuuint64_t*>(strides),
            reinterpret_cast<const cuuint32_t*>(box), elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t proj_tma_smem_bytes(bool absorb, int Dn, int Vd) {
  const int w_rows = absorb ? Dn : Vd;
  const int a_chunks = absorb ? Dn / 64 : 8;
  return (size_t)(absorb ? 4 : 8) * w_rows * 128 + (size_t)a_chunks * kTRows * 128 + 128 + 1024;
}

cudaError_t launch_proj_tma(bool absorb, const void* act, const void* w, void* out, int B, int H, int Q,
                            int Dn, int Vd, int Ckv, cudaStream_t st) {
  ProjTmaArgs a;
  memset(&a, 0, sizeof(a));
  a.out = reinterpret_cast<__nv_bfloat16*>(out);
  a.H = H;
  a.Q = Q;
  a.rows = B * Q;
  a.Dn = Dn;
  a.Vd = Vd;
  a.w_row0 = absorb ? 0 : Dn;
  a.w_rows = absorb ? Dn : Vd;
  a.a_chunks = absorb ? Dn / 64 : Ckv / 64;
  a.out_cols = absorb ? Ckv : Vd;
  {
    // wkv_b rows of all heads, 8 chunks of 64 columns
    uint64_t d[3] = {64, (uint64_t)H * (Dn + Vd), 8};
    uint64_t s[2] = {(uint64_t)Ckv * 2, 128};
    uint32_t bx[3] = {64, (uint32_t)a.w_rows, 1};
    if (!proj_encode(&a.tm_w, w, 3, d, s, bx)) return cudaErrorInvalidValue;
  }
  {
    // activation (B, H, Q, cols) as (64, Q, B, chunks, H): a box of 64/Q
    // sequences lands as [chunk][row n = b*Q + q][128 B]
    const uint64_t cols = absorb ? Dn : Ckv;
    uint64_t d[5] = {64, (uint64_t)Q, (uint64_t)B, cols / 64, (uint64_t)H};
    uint64_t s[4] = {cols * 2, (uint64_t)H * Q * cols * 2, 128, (uint64_t)Q * cols * 2};
    uint32_t bx[5] = {64, (uint32_t)Q, (uint32_t)(kTRows / Q), (uint32_t)(cols / 64), 1};
    if (!proj_encode(&a.tm_a, act, 5, d, s, bx)) return cudaErrorInvalidValue;
  }
  const int smem = (int)proj_tma_smem_bytes(absorb, Dn, Vd);
  auto kern = absorb ? proj_tma_kernel<true> : proj_tma_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(H, (a.rows + kTRows - 1) / kTRows, absorb ? 2 : 1);
  cfg.blockDim = dim3(kTThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

size_t proj_smem_bytes(bool absorb, int Dn, int Vd, int Ckv) {
  const int w_rows = absorb ? Dn : Vd;
  const int K = absorb ? Dn : Ckv;
  const int w_blocks = absorb ? 4 : 8;
  return (size_t)w_blocks * w_rows * 128 + (size_t)(K / 64) * kRowsPerCta * 128 + 64 + 1024;
}

cudaError_t launch_proj(bool absorb, const void* act, const void* w, void* out, int B, int H, int Q,
                        int Dn, int Vd, int Ckv, cudaStream_t st) {
  ProjArgs a;
  a.act = reinterpret_cast<const __nv_bfloat16*>(act);
  a.w = reinterpret_cast<const __nv_bfloat16*>(w);
  a.out = reinterpret_cast<__nv_bfloat16*>(out);
  a.H = H;
  a.Q = Q;
  a.rows = B * Q;
  a.w_head_rows = Dn + Vd;
  a.w_row0 = absorb ? 0 : Dn;
  a.w_rows = absorb ? Dn : Vd;
  a.K = absorb ? Dn : Ckv;
  a.out_cols = absorb ? Ckv : Vd;
  a.w_units = absorb ? 32 : 64;
  a.absorb = absorb ? 1 : 0;
  a.err = nullptr;
  const int smem = (int)proj_smem_bytes(absorb, Dn, Vd, Ckv);
  auto kern = absorb ? proj_sm100_kernel<true> : proj_sm100_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(H, absorb ? 2 : 1, (a.rows + kRowsPerCta - 1) / kRowsPerCta);
  cfg.blockDim = dim3(kPThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool sm100_proj_supported(int B, int H, int Q, int Dn, int Vd, int Ckv, const void* act,
                          const void* w, const void* out) {
  if (B < 1 || H < 1 || Q < 1) return false;
  // Ckv = 512 (8 blocks of 64), Vd = 128 (one M tile), Dn in {64, 128}: the
  // whole slice and 64 rows fit in shared memory and in 24 loads per thread
  if (Ckv != 512 || Vd != 128 || !(Dn == 64 || Dn == 128)) return false;
  const auto aligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!aligned(act) || !aligned(w) || !aligned(out)) return false;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return false;
  return major == 10;
}

// The TMA-fed kernel takes Q in {1, 2, 4} (a 64-row block holds whole
// sequences) and 16-byte aligned row strides; other shapes take the
// register-staged kernel.
static bool proj_tma_ok(int Q, const void* act, const void* w) {
  return (Q == 1 || Q == 2 || Q == 4) && (reinterpret_cast<uintptr_t>(act) & 15u) == 0 &&
         (reinterpret_cast<uintptr_t>(w) & 15u) == 0 && proj_encode_fn() != nullptr;
}

cudaError_t launch_absorb_sm100(const void* q_nope, const void* wkv_b, void* q_lat, int B, int H,
                                int Q, int Dn, int Vd, int Ckv, cudaStream_t st) {
  if (proj_tma_ok(Q, q_nope, wkv_b))
    return launch_proj_tma(true, q_nope, wkv_b, q_lat, B, H, Q, Dn, Vd, Ckv, st);
  return launch_proj(true, q_nope, wkv_b, q_lat, B, H, Q, Dn, Vd, Ckv, st);
}

cudaError_t launch_up_proj_sm100(const void* x, const void* wkv_b, void* out, int B, int H, int Q,
                                 int Dn, int Vd, int Ckv, cudaStream_t st) {
  if (proj_tma_ok(Q, x, wkv_b))
    return launch_proj_tma(false, x, wkv_b, out, B, H, Q, Dn, Vd, Ckv, st);
  return launch_proj(false, x, wkv_b, out, B, H, Q, Dn, Vd, Ckv, st);
}

}  // namespace mla
