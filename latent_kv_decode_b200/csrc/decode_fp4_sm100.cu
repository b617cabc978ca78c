// Tensor-core decode for the shared-latent FP4 cache (the openarchlab
// DeepSeek-V4.1-Flash page, sections on the 288-byte latent entry and the
// attention sink): K = V = the 512-wide latent, dequantised from E2M1 codes
// with one E4M3 scale per 16 channels; the softmax denominator takes the sink
// logit once; x's last 64 dims are rotated back by the query position.
//
// One CTA per (64-row query block, sequence, split); 1-SM tcgen05 MMAs with
// M = 64 (the query block). Per 64-token tile:
//
//   load       two bulk copies of 32 contiguous 288-byte entries (a page of
//              64 tokens holds both halves), plus L2 prefetches two tiles ahead
//   dequant    8 warps decode each entry to 512 bf16 with byte permutes (no
//              tables) into a tile stored in the 128-byte-swizzled layout the
//              MMAs read: K-major rows for S = Q . K^T, and the same bytes as
//              the MN-major V of O += P.V (one tile serves both, so every entry
//              is read once). Every E2M1 x E4M3 product is exact in bf16. Rows
//              past the sequence are stored as zeros.
//   S = Q.K^T  M = 64, N = 64, K = 512 (32 MMAs of K = 16). An MMA costs about
//              the same at N = 32 and N = 64, so the wider tile halves the
//              tensor-pipe time per token of this step.
//   softmax    one lane per row (lanes 0-15 of each TMEM subpartition hold an
//              M = 64 result), base 2, lazy rescale (threshold 2^8)
//   O += P.V   2 MMAs of N = 256 per 16 tokens; the first 256 columns of O
//              sit in lanes 0-15 of each subpartition, the second 256 in
//              lanes 16-31 (the interleaved M = 64 placement), so O takes
//              256 TMEM columns and the two S buffers 128 more.
//
// Shared memory (219 KB): Q 64 KB; bf16 tile ring 2 x 64 KB; entry ring
// 2 x 9 KB (32-token halves); P 8 KB (128-byte swizzle).
//
// Warp roles (448 threads): warp 0 loader (Q, entries), warp 1 MMA issuer and
// TMEM owner, warps 2-9 dequant, warps 10-13 softmax + epilogue. Every wait is
// bounded; a timeout sets MLA_DEVICE_ERR_TIMEOUT and the kernel unwinds.
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "common.cuh"
#include "launch.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kThreads = 448;
constexpr int kDeqWarps = 8;
constexpr int kLoaderWarp = 0, kMmaWarp = 1, kDeqWarp0 = 2, kSoftWarp0 = kDeqWarp0 + kDeqWarps;
constexpr int kTT = 64;                     // tokens per tile
constexpr int kHalf = 32;                   // tokens per entry copy
constexpr int kRows = 64;                   // query rows per CTA
constexpr int kEntry = 288;                 // bytes per FP4 entry (512 codes + 32 scales)
constexpr int kRawStages = 2;
constexpr int kRawStage = kHalf * kEntry;   // 9216 B
constexpr int kKStages = 2;
constexpr int kKChunk = kTT * 128;          // 64 rows x 64 dims bf16 (8 KB)
constexpr int kKStage = 8 * kKChunk;        // 64 KB
constexpr int kPBuf = kRows * kTT * 2;      // 8 KB, 128-byte rows
constexpr int kSBufs = 2;
constexpr int kPrefetchHalves = 4;          // L2 prefetch distance (two tiles)

constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + 8 * 8192;
constexpr int kOffRaw = kOffK + kKStages * kKStage;
constexpr int kOffP = kOffRaw + kRawStages * kRawStage;
constexpr int kOffBar = kOffP + kPBuf;
enum : int {
  B_QFULL = 0,
  B_RAWFULL = B_QFULL + 1,
  B_RAWEMPTY = B_RAWFULL + kRawStages,
  B_KFULL = B_RAWEMPTY + kRawStages,
  B_KEMPTY = B_KFULL + kKStages,
  B_SFULL = B_KEMPTY + kKStages,
  B_SFREE = B_SFULL + kSBufs,
  B_PFULL = B_SFREE + kSBufs,
  B_PVDONE = B_PFULL + 1,
  B_COUNT = B_PVDONE + 1
};
constexpr int kOffTmemPtr = kOffBar + B_COUNT * 8;
constexpr int kOffAbort = kOffTmemPtr + 4;
constexpr int kSmemBytes = kOffBar + 512;
constexpr int kSmemAlloc = kSmemBytes + 1024;
static_assert(kOffAbort + 4 <= kSmemBytes, "barrier area overflow");
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(kOffK % 1024 == 0 && kOffP % 1024 == 0 && kOffRaw % 16 == 0, "operand alignment");
static_assert(kTile % kTT == 0, "split ranges start on tile boundaries");

constexpr uint32_t kColO = 0;               // O: columns 0-255, lanes 0-15 (dims 0-255) and 16-31 (256-511)
constexpr uint32_t kColS = 256;             // S buffer i at columns 256 + 64 i, lanes 0-15
constexpr uint32_t kTmemCols = 512;

constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

struct alignas(64) Fp4Params {
  CUtensorMap tm_q;   // q (B*HQ, 512) bf16, box 64 x 64
  DecodeParams p;
  int paged;
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Byte permute with the sign-replicating selector mode (selector bit 3).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Eight E2M1 codes (byte k of x holds channel 2k in its low nibble and 2k+1
// in its high nibble) to four bf16x2 words, exactly. The bf16 patterns of
// the eight magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 are split into a low-byte
// and a high-byte table of 8 bytes each, indexed by the magnitude bits with
// prmt; the sign byte is 0x80 or 0 from prmt's sign replication of the byte
// whose top bit is the nibble's sign bit (x << 4 for even nibbles, x for odd).
__device__ __forceinline__ void e2m1x8_to_bf16x2(uint32_t x, uint32_t (&w)[4]) {
  constexpr uint32_t kLo03 = 0xC0800000u, kLo47 = 0xC0804000u;   // 00 00 80 C0 | 00 40 80 C0
  constexpr uint32_t kHi03 = 0x3F3F3F00u, kHi47 = 0x40404040u;   // 00 3F 3F 3F | 40 40 40 40
  const uint32_t x4 = x << 4;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t sel = (h ? (x >> 16) : x) & 0x7777u;
    const uint32_t lo = prmt(kLo03, kLo47, sel);
    const uint32_t sg = prmt(x4, x, h ? 0xFBEAu : 0xD9C8u);
    const uint32_t hi = prmt(kHi03, kHi47, sel) | (sg & 0x80808080u);
    w[2 * h] = prmt(lo, hi, 0x5140u);       // channels 4h, 4h+1
    w[2 * h + 1] = prmt(lo, hi, 0x7362u);   // channels 4h+2, 4h+3
  }
}

// One E4M3 scale byte as bf16x2 (both halves), exactly, through the
// hardware FP8 -> f16 conversion (every E4M3 value is an f16 value).
__device__ __forceinline__ __nv_bfloat162 e4m3_to_bf16x2(uint32_t byte) {
  const __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)byte, __NV_E4M3);
  const float f = __half2float(__half(hr));
  const uint32_t w = pack_bf16(f, f);
  return *reinterpret_cast<const __nv_bfloat162*>(&w);
}

// Page table entry of token t is usable (paged caches only).
__device__ __forceinline__ bool page_ok(const DecodeParams& p, int b, int t) {
  if (!p.block_table) return true;
  const int pg = p.block_table[(int64_t)b * p.max_pages + (t >> 6)];
  return pg >= 0 && pg < p.num_pages;
}

__device__ __forceinline__ uint32_t swz128(int r, int u) {
  return (uint32_t)r * 128u + ((uint32_t)((u & 7) ^ (r & 7)) << 4);
}

// Source of the entry copy for tokens [t0, t0 + 32): the row pointer and the
// number of entries (0 past a contiguous cache's end). A paged copy never
// crosses a page (t0 is a multiple of 32, pages hold 64 tokens); a bad page
// reads page 0, and the softmax masks its tokens.
__device__ __forceinline__ const uint8_t* entry_src(const Fp4Params& P, const uint8_t* kvb, int b, int len,
                                                    int t0, int& n, bool& bad) {
  const DecodeParams& p = P.p;
  bad = false;
  if (P.paged) {
    int pg = 0;
    if (t0 < len) {
      pg = p.block_table[(int64_t)b * p.max_pages + (t0 >> 6)];
      if (pg < 0 || pg >= p.num_pages) {
        bad = true;
        pg = 0;
      }
    }
    n = kHalf;
    return kvb + ((int64_t)pg * 64 + (t0 & 63)) * kEntry;
  }
  n = min(kHalf, p.Lk - t0);
  return kvb + (int64_t)b * p.kv_batch + (int64_t)(n > 0 ? t0 : 0) * kEntry;
}

__global__ void __launch_bounds__(kThreads, 1) decode_fp4_sm100_kernel(const __grid_constant__ Fp4Params P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb0 = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sb0 - raw);
  const DecodeParams& p = P.p;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rb = blockIdx.x, b = blockIdx.y, z = blockIdx.z;
  auto bar = [&](int i) -> uint32_t { return sb0 + kOffBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    for (int s = 0; s < kRawStages; ++s) {
      mbar_init(bar(B_RAWFULL + s), 1);
      mbar_init(bar(B_RAWEMPTY + s), kDeqWarps);   // one arrival per dequant warp
    }
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(B_KFULL + s), kDeqWarps);      // one arrival per dequant warp
      mbar_init(bar(B_KEMPTY + s), 1);
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_SFREE + i), 1);
    }
    mbar_init(bar(B_PFULL), 1);
    mbar_init(bar(B_PVDONE), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(sb0 + kOffTmemPtr, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmemPtr);
  // everything above overlapped the previous kernel; global inputs are read
  // only once that grid has completed
  pdl_wait();
  const int len = seq_len_of(p, b);
  int t_begin, t_end;
  split_range(len, p.num_splits, z, t_begin, t_end);
  const int ntiles = (t_end - t_begin + kTT - 1) / kTT;
  auto fail = [&]() {
    *abort_flag = 1;
    flag_error(p, MLA_DEVICE_ERR_TIMEOUT);
  };
  const uint8_t* kvb = reinterpret_cast<const uint8_t*>(p.kv);

  if (warp == kLoaderWarp) {
    // ------------------------------------------------------------------ loader
    if (lane == 0) {
      tma_prefetch_desc(&P.tm_q);
      const int qrow = b * p.HQ + rb * kRows;
      mbar_arrive_expect_tx(bar(B_QFULL), 8 * 8192);
      for (int c = 0; c < 8; ++c) tma_load_2d(sb0 + kOffQ + c * 8192, &P.tm_q, bar(B_QFULL), 64 * c, qrow);
      const int nh = 2 * ntiles;
      for (int hj = 0; hj < kPrefetchHalves && hj < nh; ++hj) {
        int n;
        bool bad;
        const uint8_t* src = entry_src(P, kvb, b, len, t_begin + kHalf * hj, n, bad);
        if (n > 0) prefetch_l2_bulk(src, (uint32_t)(n * kEntry));
      }
      bool ok = true;
      for (int hj = 0; hj < nh && ok; ++hj) {
        const int s = hj % kRawStages;
        if (hj >= kRawStages && !mbar_wait(bar(B_RAWEMPTY + s), ((hj / kRawStages) - 1) & 1)) {
          ok = false;
          break;
        }
        int n;
        bool bad;
        const uint8_t* src = entry_src(P, kvb, b, len, t_begin + kHalf * hj, n, bad);
        if (bad) flag_error(p, MLA_DEVICE_ERR_BLOCK_TABLE);
        if (n > 0) {
          mbar_arrive_expect_tx(bar(B_RAWFULL + s), (uint32_t)(n * kEntry));
          bulk_load(sb0 + kOffRaw + s * kRawStage, src, (uint32_t)(n * kEntry), bar(B_RAWFULL + s));
        } else {
          mbar_arrive(bar(B_RAWFULL + s));   // nothing left in the cache: rows are zero-filled
        }
        const int hp = hj + kPrefetchHalves;
        if (hp < nh) {
          const uint8_t* ps = entry_src(P, kvb, b, len, t_begin + kHalf * hp, n, bad);
          if (n > 0) prefetch_l2_bulk(ps, (uint32_t)(n * kEntry));
        }
        if (*abort_flag) ok = false;
      }
      if (!ok) fail();
    }
    __syncwarp();
  } else if (warp >= kDeqWarp0 && warp < kDeqWarp0 + kDeqWarps) {
    // ------------------------------------------------------------------ dequant
    // Per 32-token half: 2048 pieces of 8 channels, 8 per thread: piece i =
    // token i/64, chunk (i/8)%8, 16-byte unit i%8 (channels 64 chunk + 8 unit).
    // A warp covers one token's 4 chunks x 8 units: whole 128-byte rows, so
    // both the entry reads and the swizzled tile stores are conflict-free.
    const int dt = threadIdx.x - kDeqWarp0 * 32;   // 0..255
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      const int ks = j % kKStages;
      bool got = j < kKStages || mbar_wait(bar(B_KEMPTY + ks), ((j / kKStages) - 1) & 1);
      got = __all_sync(0xffffffffu, got) != 0;
      const uint32_t kbase = kOffK + ks * kKStage;
      for (int h = 0; h < 2 && got; ++h) {
        const int hj = 2 * j + h, rs = hj % kRawStages;
        got = mbar_wait(bar(B_RAWFULL + rs), (hj / kRawStages) & 1);
        if (!__all_sync(0xffffffffu, got)) {
          got = false;
          break;
        }
        const uint8_t* rawp = smem + kOffRaw + rs * kRawStage;
        const int t0 = t_begin + kHalf * hj;
        constexpr int kPieces = 2048 / (32 * kDeqWarps);
        uint32_t cw[kPieces], sb[kPieces];
#pragma unroll
        for (int k = 0; k < kPieces; ++k) {
          const int i = dt + 32 * kDeqWarps * k, t = i >> 6, c = (i >> 3) & 7, u = i & 7;
          const uint8_t* e = rawp + t * kEntry;
          cw[k] = *reinterpret_cast<const uint32_t*>(e + 32 * c + 4 * u);
          sb[k] = e[256 + 4 * c + (u >> 1)];
        }
#pragma unroll
        for (int k = 0; k < kPieces; ++k) {
          const int i = dt + 32 * kDeqWarps * k, t = i >> 6, c = (i >> 3) & 7, u = i & 7;
          // rows past the sequence (stale or never loaded) become zeros
          const __nv_bfloat162 s2 = (t0 + t < len) ? e4m3_to_bf16x2(sb[k]) : __float2bfloat162_rn(0.f);
          uint32_t w[4];
          e2m1x8_to_bf16x2(cw[k], w);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const __nv_bfloat162 v = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&w[q]), s2);
            w[q] = *reinterpret_cast<const uint32_t*>(&v);
          }
          *reinterpret_cast<uint4*>(smem + kbase + c * kKChunk + swz128(kHalf * h + t, u)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_RAWEMPTY + rs));
      }
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_KFULL + ks));
      if (*abort_flag) ok = false;
      ok = __all_sync(0xffffffffu, ok) != 0;
    }
    if (!ok && lane == 0) fail();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(kRows, kTT, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(kRows, 256, false, true);
      const uint64_t qd = smem_desc(sb0 + kOffQ, 16, 1024, kSwizzle128B);
      const uint64_t pd = smem_desc(sb0 + kOffP, 16, 1024, kSwizzle128B);
      bool ok = mbar_wait(bar(B_QFULL), 0);
      int qj = 0, pj = 0;
      uint64_t t_idle = global_ns();
      uint32_t idle = 0;
      while (ok && pj < ntiles) {
        bool prog = false;
        if (qj < ntiles) {
          const int sbuf = qj % kSBufs, ks = qj % kKStages;
          const bool sfree = qj < kSBufs || mbar_poll(bar(B_SFREE + sbuf), ((qj / kSBufs) - 1) & 1);
          if (sfree && mbar_poll(bar(B_KFULL + ks), (qj / kKStages) & 1)) {
            tc_fence_after();
            const uint64_t kd = smem_desc(sb0 + kOffK + ks * kKStage, 16, 1024, kSwizzle128B);
            const uint32_t d = tmem + kColS + 64u * sbuf;
#pragma unroll
            for (int kk = 0; kk < 32; ++kk) {
              const int c = kk >> 2, sub = kk & 3;
              mma_bf16_ss(d, desc_advance(qd, c * 8192 + 32 * sub),
                          desc_advance(kd, c * kKChunk + 32 * sub), idesc_qk, kk > 0);
            }
            mma_commit(bar(B_SFULL + sbuf));
            ++qj;
            prog = true;
          }
        }
        if (pj < qj && mbar_poll(bar(B_PFULL), pj & 1)) {
          tc_fence_after();
          const int ks = pj % kKStages;
          const uint64_t vd = smem_desc(sb0 + kOffK + ks * kKStage, kKChunk, 1024, kSwizzle128B);
#pragma unroll
          for (int n = 0; n < 2; ++n) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              // P: 16 tokens per step (K-major, 128-byte rows); V: the tile's
              // chunks 4n..4n+3 (MN-major); D: lanes 16n.. of each subpartition
              mma_bf16_ss(tmem + ((16u * n) << 16) + kColO, desc_advance(pd, 32 * kk),
                          desc_advance(vd, 4 * n * kKChunk + 2048 * kk), idesc_pv,
                          (pj > 0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(bar(B_KEMPTY + ks));
          mma_commit(bar(B_PVDONE));
          ++pj;
          prog = true;
        }
        if (prog) {
          idle = 0;
        } else if ((++idle & 255u) == 0) {
          if (idle == 256u) t_idle = global_ns();
          else if (global_ns() - t_idle > 1000000000ull || *abort_flag) ok = false;
        }
      }
      if (!ok) fail();
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    // Warp g = warp % 4 owns TMEM subpartition g: lane i < 16 holds row
    // 16 g + i of S and the first 256 columns of its O row; lane 16 + i holds
    // the second 256 columns of the same row.
    const int g = warp & 3;
    const int hi = lane >> 4, m = 16 * g + (lane & 15);
    const int r = rb * kRows + m;
    const int q = r % p.Q;
    const int h = r / p.Q;
    const uint32_t lane_base = (uint32_t)(32 * g) << 16;
    const float sl2 = p.scale_log2;
    const uint8_t* mask = p.mask;
    const bool causal = p.causal != 0;
    const int causal_last = len - p.Q + q;
    const bool paged = p.block_table != nullptr;
    const bool leader = (warp == kSoftWarp0 && lane == 0);
    float m_run = -INFINITY, l_run = 0.f;
    bool ab = false;
    auto wait_pv = [&](int t) {
      if (!ab) ab = !mbar_wait(bar(B_PVDONE), t & 1);
    };
    for (int j = 0; j < ntiles; ++j) {
      const int sbuf = j % kSBufs;
      if (!ab) ab = !mbar_wait(bar(B_SFULL + sbuf), (j / kSBufs) & 1);
      ab = __any_sync(0xffffffffu, ab);
      float s[kTT];
      if (!ab) {
        tc_fence_after();
        uint32_t v[4][16];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld16(tmem + lane_base + kColS + 64u * sbuf + 16u * c, v[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 16; ++i) s[16 * c + i] = __uint_as_float(v[c][i]);
      } else {
#pragma unroll
        for (int i = 0; i < kTT; ++i) s[i] = 0.f;
      }
      tc_fence_before();
      named_bar_sync(1, 128);   // every warp has read S(j)
      if (leader) mbar_arrive(bar(B_SFREE + sbuf));

      const int tb = t_begin + j * kTT;
      int lim = t_end - tb;
      if (causal) lim = min(lim, causal_last - tb + 1);
      if (paged && !page_ok(p, b, tb < len ? tb : 0)) lim = 0;   // a tile is one page
      if (ab) lim = 0;
      // visibility of the tile's 64 tokens as bit masks: the question's mask
      // is read once per token, one lane each (tb is the same for every row)
      uint32_t v0 = lim >= 32 ? 0xffffffffu : (lim <= 0 ? 0u : (1u << lim) - 1u);
      uint32_t v1 = lim >= 64 ? 0xffffffffu : (lim <= 32 ? 0u : (1u << (lim - 32)) - 1u);
      if (mask != nullptr) {
        v0 &= __ballot_sync(0xffffffffu, tb + lane < t_end && mask[tb + lane] != 0);
        v1 &= __ballot_sync(0xffffffffu, tb + 32 + lane < t_end && mask[tb + 32 + lane] != 0);
      }
      // eight independent partial maxima and sums keep the dependency chains short
      float mp[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mp[i] = -INFINITY;
#pragma unroll
      for (int c = 0; c < kTT; ++c) {
        const uint32_t vb = c < 32 ? v0 : v1;
        s[c] = ((vb >> (c & 31)) & 1u) ? s[c] * sl2 : -INFINITY;
        mp[c & 7] = fmaxf(mp[c & 7], s[c]);
      }
      const float mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                             fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
      const float m_new = fmaxf(m_run, mx);
      const bool need = (m_new - m_run) > kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = exp2f(m_run - m_new);
        m_run = m_new;
      }
      uint32_t pk[kTT / 2];
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
      const bool none = (m_run == -INFINITY);
#pragma unroll
      for (int c = 0; c < kTT / 2; ++c) {
        const float p0 = none ? 0.f : fast_exp2(s[2 * c] - m_run);
        const float p1 = none ? 0.f : fast_exp2(s[2 * c + 1] - m_run);
        ps[c & 3] += p0 + p1;
        pk[c] = pack_bf16(p0, p1);
      }
      l_run = l_run * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
      // lanes 16-31 rescale the second half of the same rows: take lane i's alpha
      const float alpha_row = __shfl_sync(0xffffffffu, alpha, lane & 15);
      const bool need_row = __shfl_sync(0xffffffffu, need, lane & 15);

      // P and O are free once PV(j - 1) has completed
      if (j >= 1) wait_pv(j - 1);
      if (hi == 0) {
        uint8_t* prow = smem + kOffP + m * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(prow + 16 * (c ^ (m & 7))) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      if (__any_sync(0xffffffffu, need_row && j > 0)) {
        ab = __any_sync(0xffffffffu, ab);
        if (!ab) {
          tc_fence_after();
          // 256 columns in 4 rounds of 64: four loads per wait
#pragma unroll 1
          for (int c = 0; c < 16; c += 4) {
            uint32_t v[4][16];
            const uint32_t ta = tmem + lane_base + kColO + 16u * c;
#pragma unroll
            for (int k = 0; k < 4; ++k) tmem_ld16(ta + 16u * k, v[k]);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 4; ++k) {
#pragma unroll
              for (int i = 0; i < 16; ++i) v[k][i] = __float_as_uint(__uint_as_float(v[k][i]) * alpha_row);
              tmem_st16(ta + 16u * k, v[k]);
            }
          }
          tmem_wait_st();
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(1, 128);   // P(j) of every row is written
      if (leader) mbar_arrive(bar(B_PFULL));
    }

    // ---------------------------------------------------------------- epilogue
    if (ntiles > 0) wait_pv(ntiles - 1);
    ab = __any_sync(0xffffffffu, ab);
    if (ab && lane == 0) fail();
    tc_fence_after();
    const bool have_o = ntiles > 0 && !ab;
    const float mrow = __shfl_sync(0xffffffffu, m_run, lane & 15);
    const float lrow = __shfl_sync(0xffffffffu, l_run, lane & 15);
    const int64_t grow = (int64_t)b * p.HQ + r;
    float scale_o, lse;
    if (p.num_splits > 1) {
      scale_o = lrow > 0.f ? 1.f / lrow : 0.f;
      lse = lrow > 0.f ? (mrow + log2f(lrow)) * kLn2 : -INFINITY;
    } else {
      float mfin = mrow, lfin = lrow, w = 1.f;
      if (p.sinks) {
        const float sk = p.sinks[h] * kLog2e;
        const float m2 = fmaxf(mrow, sk);
        w = (mrow == -INFINITY) ? 0.f : exp2f(mrow - m2);
        lfin = lrow * w + exp2f(sk - m2);
        mfin = m2;
      }
      scale_o = lfin > 0.f ? w / lfin : 0.f;
      lse = lfin > 0.f ? (mfin + log2f(lfin)) * kLn2 : -INFINITY;
    }
    // Inverse RoPE of an unsplit row block: with Q = 1 every row of the CTA
    // sits at position len - 1, so lane j evaluates tail pair j's rotation
    // once (the double-precision angle of inverse_rope_pair) and the lanes
    // holding the tail take it by shuffle, instead of each tail lane
    // evaluating all of its pairs in turn.
    const int rope_base = p.Ckv - p.rope_tail;
    const bool rope_shared = p.num_splits == 1 && p.rope_tail > 0 && p.rope_tail <= 64 && p.Q == 1;
    double rope_c = 1.0, rope_s = 0.0;
    if (rope_shared && 2 * lane < p.rope_tail) {
      const double freq = pow((double)p.rope_theta, -2.0 * (double)lane / (double)p.rope_tail);
      sincos(-(double)(len - 1) * freq, &rope_s, &rope_c);
    }
#pragma unroll 1
    for (int c = 0; c < 16; ++c) {
      uint32_t v[16];
      if (have_o) {
        tmem_ld16(tmem + lane_base + kColO + 16u * c, v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0u;
      }
      float f[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) f[i] = __uint_as_float(v[i]) * scale_o;
      const int col = 256 * hi + 16 * c;
      if (p.num_splits > 1) {
        float* o = p.ws_o + ((int64_t)z * p.B * p.HQ + grow) * p.Ckv + col;
#pragma unroll
        for (int i = 0; i < 16; i += 4)
          *reinterpret_cast<float4*>(o + i) = make_float4(f[i], f[i + 1], f[i + 2], f[i + 3]);
      } else {
        if (rope_shared) {
          if (256 + 16 * c + 16 > rope_base) {   // the same test in every lane: all shuffle
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
              const int cc = col + i;
              const int jp = cc >= rope_base ? (cc - rope_base) >> 1 : 0;
              const double cr = __shfl_sync(0xffffffffu, rope_c, jp);
              const double sr = __shfl_sync(0xffffffffu, rope_s, jp);
              if (cc >= rope_base) {
                const float fa = f[i], fb = f[i + 1];
                f[i] = (float)(fa * cr - fb * sr);
                f[i + 1] = (float)(fa * sr + fb * cr);
              }
            }
          }
        } else if (p.rope_tail > 0 && col >= rope_base) {
          const int pos = len - p.Q + q;
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            const int jp = (col + i - (p.Ckv - p.rope_tail)) >> 1;
            inverse_rope_pair(f[i], f[i + 1], jp, p.rope_tail, p.rope_theta, pos);
          }
        }
        uint32_t w4[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w4[i] = pack_bf16(f[2 * i], f[2 * i + 1]);
        uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.x) + grow * p.Ckv + col);
        o[0] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        o[1] = make_uint4(w4[4], w4[5], w4[6], w4[7]);
      }
    }
    if (hi == 0) {
      if (p.num_splits > 1)
        p.ws_lse[(int64_t)z * p.B * p.HQ + grow] = lse;
      else if (p.lse)
        p.lse[grow] = lse;
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 fp4_encode_fn() {
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

}  // namespace

bool sm100_fp4_decode_supported(const mla_decode_args* a) {
  if (a->cache_dtype != MLA_FP4_E2M1_E4M3x16 || a->q_dtype != MLA_BF16) return false;
  if (a->Ckv != 512 || a->Dr != 0) return false;
  if ((a->H * a->Q) % kRows != 0) return false;
  if (a->kv_row_stride != kEntry) return false;            // contiguous entries: one bulk copy per tile
  if (a->block_table) {
    if (a->page_size != 64) return false;
  } else if (a->kv_batch_stride % 16 != 0) {
    return false;
  }
  if ((reinterpret_cast<uintptr_t>(a->q_lat) & 15u) || (reinterpret_cast<uintptr_t>(a->kv_cache) & 15u))
    return false;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10 && fp4_encode_fn() != nullptr;
}

int sm100_fp4_auto_splits(const mla_decode_args* a, int sms) {
  const int ctas = a->B * (a->H * a->Q / kRows);
  const int tiles = (a->Lk + kTile - 1) / kTile;
  if (ctas >= sms) return 1;
  int s = sms / ctas;
  if (s > tiles) s = tiles;
  return s < 1 ? 1 : s;
}

cudaError_t launch_decode_fp4_sm100(const DecodeParams& p, const mla_decode_args* a, cudaStream_t st) {
  Fp4Params P;
  memset(&P, 0, sizeof(P));
  P.p = p;
  P.paged = a->block_table != nullptr;
  {
    auto fn = fp4_encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    cuuint64_t d[2] = {512, (cuuint64_t)p.B * p.HQ};
    cuuint64_t s[1] = {512 * 2};
    cuuint32_t box[2] = {64, 64}, es[2] = {1, 1};
    if (fn(&P.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a->q_lat), d, s, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(decode_fp4_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemAlloc);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.HQ / kRows, p.B, p.num_splits);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_fp4_sm100_kernel, P);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mla
