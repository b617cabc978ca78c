// Tensor-core decode for bf16 caches (Ckv = 512, Dr = 64, H*Q a multiple of
// 128): blanks [2]-[4] and step 5 of mla_decode_step (the 6547.cn MLA decode
// question), with the absorbed score of the neuronix DeepSeek-V3/R1 page.
//
// One 2-CTA cluster per (128-row block, sequence, split). CTA r of the pair
// owns query rows [64r, 64r+64) of the block; every MMA is a pair MMA
// (tcgen05 cta_group::2, M = 128), so each SM computes its own 64 rows and the
// pair shares one K tile. Per 128-token tile of the cache:
//
//   S  = Q . K^T   over the 576 dims in 64-dim chunks (8 latent + 1 rope).
//                  CTA r supplies tokens [64r, 64r+64) of the tile (the N half
//                  of B), loaded as 4 stages of 2 latent chunks + 1 rope stage.
//   softmax        online, base 2, lazy rescale (the running max only moves
//                  when a score exceeds it by more than 2^8).
//   O += P . V     2 halves of 256 latent columns x 2 halves of 64 tokens.
//                  CTA r supplies latent columns [128r, 128r+128) of each half
//                  for all 128 tokens.
//
// The latent rows are therefore read twice per tile (once as K, once as V,
// cut differently between the pair); the V read follows the K read of the
// same rows closely enough to hit in L2, so HBM sees each cache row once (an
// explicit L2 prefetch ahead of the K producer measured no gain and is off,
// kPrefetchTiles = 0). Every TMA request moves 64 rows x 2 chunks
// (16 KB) through a 4-D view of the cache whose box lands already in the
// 128-byte-swizzled layout the MMAs read. Scores and the output accumulator
// live in TMEM (S double-buffered: 2 x 64 columns; O: 2 x 128 columns).
//
// Warp roles (224 threads): warp 0 K producer (+ Q), warp 1 MMA issuer (even
// CTA only) and TMEM owner, warps 2-5 softmax + epilogue (TMEM lane =
// 32*(warp%4) + lane), warp 6 V producer. Every wait is bounded; a timeout sets
// MLA_DEVICE_ERR_TIMEOUT and the kernel unwinds.
#include <cudaTypedefs.h>
#include <math.h>

#include "common.cuh"
#include "launch.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kThreads = 224;
constexpr int kTileT = 128;                 // tokens per tile (both CTAs)
constexpr int kKStages = 3;                 // ring of K stages: 3 chunks of 64 dims (24 KB); a tile
constexpr int kKStage = 24576;
constexpr int kVStages = 4;                 // ring of V stages (16 KB): a tile
constexpr int kStage = 16384;               // V stage bytes per CTA
constexpr int kKUses = 3;                   // K stage uses per tile: chunks 0-2, 3-5, 6-7 + rope
constexpr int kPrefetchTiles = 0;           // L2 prefetch distance of the K producer (off: measured no gain)
constexpr int kQBlocks = 9;                 // 64-dim blocks of the 576-wide query row
constexpr int kQBytes = kQBlocks * 8192;    // 64 rows x 128 B per block
constexpr int kPBuf = 16384;                // P: 64 rows x 128 tokens bf16 (2 blocks), one buffer

constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;
constexpr int kOffV = kOffK + kKStages * kKStage;
constexpr int kOffP = kOffV + kVStages * kStage;
constexpr int kOffBar = kOffP + kPBuf;
enum : int {
  B_KFULL = 0,
  B_KEMPTY = B_KFULL + kKStages,
  B_VFULL = B_KEMPTY + kKStages,
  B_VEMPTY = B_VFULL + kVStages,
  B_QFULL = B_VEMPTY + kVStages,
  B_SFULL = B_QFULL + 1,
  B_SFREE = B_SFULL + 2,
  B_PFULL = B_SFREE + 2,
  B_PVDONE = B_PFULL + 2,
  B_COUNT = B_PVDONE + 2
};
constexpr int kOffTmemPtr = kOffBar + B_COUNT * 8;
constexpr int kOffAbort = kOffTmemPtr + 4;
constexpr int kOffXchg = kOffBar + 512;     // float xmax[2][128], xsum[128]
constexpr int kSmemBytes = kOffXchg + 3 * 128 * 4;
constexpr int kSmemAlloc = kSmemBytes + 1024;

constexpr uint32_t kColS = 0;               // S buffers at columns 0 and 64
constexpr uint32_t kColO = 128;             // O halves at columns 128 and 256
constexpr uint32_t kTmemCols = 512;

constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

struct alignas(64) Sm100Params {
  CUtensorMap tm_q;    // q_lat  (B*HQ, 512), box 64 x 64
  CUtensorMap tm_qpe;  // q_pe   (B*HQ, 64),  box 64 x 64
  CUtensorMap tm_k;    // latent cache as (64 dims, rows, 8 chunks, seq|page): box 64 rows x 2 chunks
  CUtensorMap tm_k3;   // the same view, box 64 rows x 3 chunks
  CUtensorMap tm_pe;   // rope cache (64 dims, rows, seq|page): box 64 rows
  DecodeParams p;
  int paged;
};

// 2^x on the SFU; subnormal results flush to zero (probabilities below
// 2^-126 of the row maximum are irrelevant at bf16 precision).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ bool bar_or(int id, int count, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "barrier.red.or.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return out != 0;
}

// Pool page of token t of sequence b (page size 64), 0 for tokens past the
// end; a bad table entry is flagged and replaced by page 0 (its tokens are
// masked by the softmax).
__device__ __forceinline__ int page_of(const DecodeParams& p, int b, int t, int len) {
  if (t >= len) return 0;
  const int pg = p.block_table[(int64_t)b * p.max_pages + (t >> 6)];
  if (pg < 0 || pg >= p.num_pages) {
    flag_error(p, MLA_DEVICE_ERR_BLOCK_TABLE);
    return 0;
  }
  return pg;
}

__device__ __forceinline__ bool page_ok(const DecodeParams& p, int b, int t) {
  if (!p.block_table) return true;
  const int pg = p.block_table[(int64_t)b * p.max_pages + (t >> 6)];
  return pg >= 0 && pg < p.num_pages;
}

__global__ void __launch_bounds__(kThreads, 1) decode_sm100_kernel(const __grid_constant__ Sm100Params P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb0 = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sb0 - raw);
  const DecodeParams& p = P.p;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int rb = blockIdx.x >> 1, b = blockIdx.y, z = blockIdx.z;
  pdl_launch_dependents();
  auto bar = [&](int i) -> uint32_t { return sb0 + kOffBar + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
    }
    mbar_init(bar(B_QFULL), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_SFREE + i), 2);   // one arrival per CTA
      mbar_init(bar(B_PFULL + i), 2);   // one arrival per CTA
      mbar_init(bar(B_PVDONE + i), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_2sm(sb0 + kOffTmemPtr, kTmemCols);
    tmem_relinquish_2sm();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmemPtr);
  // the setup above overlapped the previous kernel (the absorb); global
  // inputs (q_lat, lengths, tables, the cache) are read only once it completed
  pdl_wait();
  const int len = seq_len_of(p, b);
  int t_begin, t_end;
  split_range(len, p.num_splits, z, t_begin, t_end);
  const int ntiles = (t_end - t_begin + kTileT - 1) / kTileT;

  auto fail = [&]() {
    *abort_flag = 1;
    flag_error(p, MLA_DEVICE_ERR_TIMEOUT);
  };
  // let copies already issued land before this CTA's shared memory goes away
  auto settle = []() {
    const uint64_t t0 = global_ns();
    while (global_ns() - t0 < 50000ull) {
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ K producer
    // Q once, then for every tile the 9 K chunks (this CTA's 64 tokens x 64 dims).
    if (lane == 0) {
      tma_prefetch_desc(&P.tm_q);
      tma_prefetch_desc(&P.tm_qpe);
      tma_prefetch_desc(&P.tm_k);
      tma_prefetch_desc(&P.tm_k3);
      tma_prefetch_desc(&P.tm_pe);
      const int qrow = b * p.HQ + rb * 128 + (int)rank * 64;
      const uint32_t qbar = map_to_rank(bar(B_QFULL), 0);
      if (rank == 0) mbar_arrive_expect_tx(bar(B_QFULL), 2 * kQBytes);
      for (int c = 0; c < 8; ++c) tma_load_2d_2sm(sb0 + kOffQ + c * 8192, &P.tm_q, qbar, 64 * c, qrow);
      tma_load_2d_2sm(sb0 + kOffQ + 8 * 8192, &P.tm_qpe, qbar, 0, qrow);
      // L2 prefetch of this CTA's 64 cache rows of a tile (latent and rope rows
      // as whole contiguous ranges), kPrefetchTiles ahead of the shared-memory loads
      auto prefetch_tile = [&](int jt) {
        const int t = t_begin + jt * kTileT + (int)rank * 64;
        if (jt >= ntiles || t >= len) return;
        const int rows = min(64, len - t);
        const char* kvb = reinterpret_cast<const char*>(p.kv);
        const char* peb = reinterpret_cast<const char*>(p.pe);
        if (P.paged) {
          const int64_t row0 = (int64_t)page_of(p, b, t, len) * 64;
          kvb += row0 * p.kv_row * 2;
          peb += row0 * p.pe_row * 2;
        } else {
          kvb += ((int64_t)b * p.kv_batch + (int64_t)t * p.kv_row) * 2;
          peb += ((int64_t)b * p.pe_batch + (int64_t)t * p.pe_row) * 2;
        }
        // the range ends at the last row's own data (strided rows may share a buffer)
        prefetch_l2_bulk(kvb, (uint32_t)(((int64_t)(rows - 1) * p.kv_row + p.Ckv) * 2));
        prefetch_l2_bulk(peb, (uint32_t)(((int64_t)(rows - 1) * p.pe_row + p.Dr) * 2));
      };
      for (int jt = 0; jt < kPrefetchTiles; ++jt) prefetch_tile(jt);
      uint32_t it = 0;
      bool ok = true;
      for (int j = 0; j < ntiles && ok; ++j) {
        if (kPrefetchTiles > 0) prefetch_tile(j + kPrefetchTiles);
        const int t = t_begin + j * kTileT + (int)rank * 64;
        int y = t, zc = b;
        if (P.paged) {
          zc = page_of(p, b, t, len);
          y = 0;
        }
        for (int u = 0; u < kKUses; ++u, ++it) {
          const uint32_t s = it % kKStages, round = it / kKStages;
          if (round > 0 && !mbar_wait_cluster(bar(B_KEMPTY + s), (round - 1) & 1)) { ok = false; break; }
          const uint32_t dst = sb0 + kOffK + s * kKStage, fb = map_to_rank(bar(B_KFULL + s), 0);
          if (rank == 0) mbar_arrive_expect_tx(bar(B_KFULL + s), 2 * kKStage);
          if (u < 2) {
            tma_load_4d_2sm(dst, &P.tm_k3, fb, 0, y, 3 * u, zc);
          } else {
            tma_load_4d_2sm(dst, &P.tm_k, fb, 0, y, 6, zc);
            tma_load_3d_2sm(dst + 2 * 8192, &P.tm_pe, fb, 0, y, zc);
          }
        }
        if (*abort_flag) ok = false;
      }
      if (!ok) {
        fail();
        settle();
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    // ------------------------------------------------------------------ V producer
    // For tile j, after QK(j) has completed (these rows sit in L2): for each
    // 256-column half and each 64-token half, this CTA's 128 latent columns.
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int j = 0; j < ntiles && ok; ++j) {
        if (!mbar_wait_cluster(bar(B_SFULL + (j & 1)), (j >> 1) & 1)) { ok = false; break; }
        const int tj = t_begin + j * kTileT;
        for (int n = 0; n < 2 && ok; ++n) {
          for (int th = 0; th < 2; ++th, ++it) {
            const int t = tj + 64 * th;
            int y = t, zc = b;
            if (P.paged) {
              zc = page_of(p, b, t, len);
              y = 0;
            }
            const uint32_t s = it % kVStages, round = it / kVStages;
            if (round > 0 && !mbar_wait_cluster(bar(B_VEMPTY + s), (round - 1) & 1)) { ok = false; break; }
            if (rank == 0) mbar_arrive_expect_tx(bar(B_VFULL + s), 2 * kStage);
            const uint32_t dst = sb0 + kOffV + s * kStage, fb = map_to_rank(bar(B_VFULL + s), 0);
            tma_load_4d_2sm(dst, &P.tm_k, fb, 0, y, 4 * n + 2 * (int)rank, zc);
          }
        }
        if (*abort_flag) ok = false;
      }
      if (!ok) {
        fail();
        settle();
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (even CTA)
    // Two independent streams, polled: QK(j) (needs S(j-2) released and K
    // stages) and PV(j) (needs P(j) and V stages). Neither waits on the other,
    // so a V stage in flight never stalls the K ring and vice versa.
    if (rank == 0 && lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(128, 256, false, true);
      const uint64_t qd0 = smem_desc(sb0 + kOffQ, 16, 1024, kSwizzle128B);
      const uint64_t kd0 = smem_desc(sb0 + kOffK, 16, 1024, kSwizzle128B);
      const uint64_t pd0 = smem_desc(sb0 + kOffP, 16, 1024, kSwizzle128B);
      const uint64_t vd0 = smem_desc(sb0 + kOffV, 8192, 1024, kSwizzle128B);
      bool ok = mbar_wait_cluster(bar(B_QFULL), 0);
      uint32_t kit = 0, vit = 0;
      int qj = 0, qu = 0;   // next QK: tile, stage use (4 latent pairs + rope)
      int pj = 0, pu = 0;   // next PV: tile, stage use (n * 2 + token half)
      uint64_t t_idle = global_ns();
      uint32_t idle = 0;
      while (ok && pj < ntiles) {
        bool prog = false;
        if (qj < ntiles) {
          const int sbuf = qj & 1;
          const bool sfree = qu > 0 || qj < 2 || mbar_poll_cluster(bar(B_SFREE + sbuf), ((qj - 2) >> 1) & 1);
          const uint32_t s = kit % kKStages;
          if (sfree && mbar_poll_cluster(bar(B_KFULL + s), (kit / kKStages) & 1)) {
            tc_fence_after();
            const uint32_t d = tmem + kColS + 64u * sbuf;
            // Q's 64-dim blocks 3 qu .. 3 qu + 2 (block 8 = rope) against the stage's three
            const uint64_t qd = desc_advance(qd0, 3 * qu * 8192);
            const uint64_t kd = desc_advance(kd0, s * kKStage);
#pragma unroll
            for (int cc = 0; cc < 3; ++cc) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                mma_bf16_ss_2sm(d, desc_advance(qd, cc * 8192 + 32 * k), desc_advance(kd, cc * 8192 + 32 * k),
                                idesc_qk, (qu | cc | k) != 0);
              }
            }
            mma_commit_2sm_mc(bar(B_KEMPTY + s), 3);
            ++kit;
            if (++qu == kKUses) {
              mma_commit_2sm_mc(bar(B_SFULL + sbuf), 3);
              qu = 0;
              ++qj;
            }
            prog = true;
          }
        }
        if (pj < qj) {
          const bool pready = pu > 0 || mbar_poll_cluster(bar(B_PFULL + (pj & 1)), (pj >> 1) & 1);
          const uint32_t s = vit % kVStages;
          if (pready && mbar_poll_cluster(bar(B_VFULL + s), (vit / kVStages) & 1)) {
            tc_fence_after();
            const int n = pu >> 1, th = pu & 1;
            const uint64_t pd = desc_advance(pd0, th * 8192);
            const uint64_t vd = desc_advance(vd0, s * kStage);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              // P: K-block th (64 tokens), 16 tokens per step; V: 2 blocks of 64 columns
              mma_bf16_ss_2sm(tmem + kColO + 128u * n, desc_advance(pd, 32 * k), desc_advance(vd, 2048 * k),
                              idesc_pv, (pj > 0 || th > 0 || k > 0) ? 1u : 0u);
            }
            mma_commit_2sm_mc(bar(B_VEMPTY + s), 3);
            ++vit;
            if (++pu == 4) {
              mma_commit_2sm_mc(bar(B_PVDONE + (pj & 1)), 3);
              pu = 0;
              ++pj;
            }
            prog = true;
          }
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
    const int g = warp & 3;
    const int L = 32 * g + lane;                // TMEM lane
    const int half = L >> 6, row = L & 63;
    const int r = rb * 128 + (int)rank * 64 + row;
    const int q = r % p.Q;
    const int h = r / p.Q;
    const uint32_t lane_base = (uint32_t)(32 * g) << 16;
    float* xmax = reinterpret_cast<float*>(smem + kOffXchg);
    float* xsum = xmax + 256;
    float m_run = -INFINITY, l_part = 0.f;
    bool ab = false;
    // loop-invariant parameters, read once into registers
    const float sl2 = p.scale_log2;
    const uint8_t* mask = p.mask;
    const bool causal = p.causal != 0;
    const int causal_last = len - p.Q + q;   // last visible token of a causal row
    const bool paged = p.block_table != nullptr;
    const bool leader_thread = (L == 0);     // arrives for this CTA on the even CTA's barriers

    for (int j = 0; j < ntiles; ++j) {
      const int sbuf = j & 1;
      float s[64];
      if (!ab) ab = !mbar_wait_cluster(bar(B_SFULL + sbuf), (j >> 1) & 1);
      ab = __any_sync(0xffffffffu, ab);
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
      }
      tc_fence_before();

      // scale to log2 units and mask: this thread holds tokens [tb, tb + 64);
      // tokens [tb, tb + lim) pass the range / causal / page tests
      const int tb = t_begin + j * kTileT + 64 * half;
      int lim = t_end - tb;
      if (causal) lim = min(lim, causal_last - tb + 1);
      if (paged && !page_ok(p, b, tb < len ? tb : 0)) lim = 0;
      if (ab) lim = 0;
      float mx = -INFINITY;
      if (mask == nullptr) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          s[c] = (c < lim) ? s[c] * sl2 : -INFINITY;
          mx = fmaxf(mx, s[c]);
        }
      } else {
        // the question's mask, one byte per lane (tb is the same across the warp)
        const uint32_t m0 = __ballot_sync(0xffffffffu, tb + lane < t_end && mask[tb + lane] != 0);
        const uint32_t m1 = __ballot_sync(0xffffffffu, tb + 32 + lane < t_end && mask[tb + 32 + lane] != 0);
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const bool vis = c < lim && (((c < 32 ? m0 : m1) >> (c & 31)) & 1u);
          s[c] = vis ? s[c] * sl2 : -INFINITY;
          mx = fmaxf(mx, s[c]);
        }
      }
      xmax[sbuf * 128 + L] = mx;
      // all four warps have read S(j) by now: release the buffer to the MMA
      const bool stop = bar_or(1, 128, ab);
      if (leader_thread) mbar_arrive_remote(map_to_rank(bar(B_SFREE + sbuf), 0));
      if (stop) {
        ab = true;
        break;
      }
      mx = fmaxf(mx, xmax[sbuf * 128 + (L ^ 64)]);
      const float m_new = fmaxf(m_run, mx);
      const bool need = (m_new - m_run) > kRescaleThreshold;
      float alpha = 1.f;
      if (need) {
        alpha = exp2f(m_run - m_new);
        m_run = m_new;
      }
      uint32_t pk[32];
      float psum = 0.f;
      const bool none = (m_run == -INFINITY);
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float p0 = none ? 0.f : fast_exp2(s[2 * c] - m_run);
        const float p1 = none ? 0.f : fast_exp2(s[2 * c + 1] - m_run);
        psum += p0 + p1;
        pk[c] = pack_bf16(p0, p1);
      }
      l_part = l_part * alpha + psum;

      // the P buffer (and O) are free once PV(j-1) is done
      if (j >= 1 && !ab) ab = !mbar_wait_cluster(bar(B_PVDONE + ((j - 1) & 1)), ((j - 1) >> 1) & 1);
      uint8_t* prow = smem + kOffP + half * 8192 + row * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 val = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow + 16 * (c ^ (row & 7))) = val;
      }
      // rescale this lane's O row when its running max moved (PV(j-1) must be done)
      const bool warp_need = __any_sync(0xffffffffu, need && j > 0);
      if (warp_need) {
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
              for (int i = 0; i < 16; ++i) v[k][i] = __float_as_uint(__uint_as_float(v[k][i]) * alpha);
              tmem_st16(ta + 16u * k, v[k]);
            }
          }
          tmem_wait_st();
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      // P(j) of all four warps is written: one arrival for this CTA
      named_bar_sync(2, 128);
      if (leader_thread) mbar_arrive_remote(map_to_rank(bar(B_PFULL + sbuf), 0));
    }

    // ---------------------------------------------------------------- epilogue
    xsum[L] = l_part;
    ab = bar_or(1, 128, ab);
    const float l_tot = l_part + xsum[L ^ 64];
    if (ntiles > 0 && !ab) ab = !mbar_wait_cluster(bar(B_PVDONE + ((ntiles - 1) & 1)), ((ntiles - 1) >> 1) & 1);
    ab = __any_sync(0xffffffffu, ab);
    if (ab) fail();
    tc_fence_after();
    const bool have_o = ntiles > 0 && !ab;
    const int64_t grow = (int64_t)b * p.HQ + r;

    float scale_o, lse;
    if (p.num_splits > 1) {
      scale_o = l_tot > 0.f ? 1.f / l_tot : 0.f;
      lse = l_tot > 0.f ? (m_run + log2f(l_tot)) * kLn2 : -INFINITY;
    } else {
      float mfin = m_run, lfin = l_tot, w = 1.f;
      if (p.sinks) {
        const float sk = p.sinks[h] * kLog2e;
        const float m2 = fmaxf(m_run, sk);
        w = (m_run == -INFINITY) ? 0.f : exp2f(m_run - m2);
        lfin = l_tot * w + exp2f(sk - m2);
        mfin = m2;
      }
      scale_o = lfin > 0.f ? w / lfin : 0.f;
      lse = lfin > 0.f ? (mfin + log2f(lfin)) * kLn2 : -INFINITY;
    }
#pragma unroll 1
    for (int n = 0; n < 2; ++n) {
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t v[16];
        if (have_o) {
          tmem_ld16(tmem + lane_base + kColO + 128u * n + 16u * c, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = 0u;
        }
        float f[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) f[i] = __uint_as_float(v[i]) * scale_o;
        const int col = 256 * n + 128 * half + 16 * c;
        if (p.num_splits > 1) {
          float* o = p.ws_o + ((int64_t)z * p.B * p.HQ + grow) * p.Ckv + col;
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(o + i) = make_float4(f[i], f[i + 1], f[i + 2], f[i + 3]);
        } else {
          if (p.rope_tail > 0 && col >= p.Ckv - p.rope_tail) {
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
    }
    if (half == 0) {
      if (p.num_splits > 1)
        p.ws_lse[(int64_t)z * p.B * p.HQ + grow] = lse;
      else if (p.lse)
        p.lse[grow] = lse;
    }
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

bool encode_bf16(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint32_t elem[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
                  reinterpret_cast<const cuuint64_t*>(dims),
                  reinterpret_cast<const cuuint64_t*>(strides_bytes),
                  reinterpret_cast<const cuuint32_t*>(box), elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool sm100_decode_supported(const mla_decode_args* a) {
  if (a->q_dtype != MLA_BF16 || a->cache_dtype != MLA_BF16) return false;
  if (a->Ckv != 512 || a->Dr != 64) return false;
  if ((a->H * a->Q) % 128 != 0) return false;
  if (a->block_table) {
    if (a->page_size != 64) return false;
  } else {
    if ((a->kv_batch_stride * 2) % 16 != 0 || (a->pe_batch_stride * 2) % 16 != 0) return false;
  }
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return false;
  return major == 10 && encode_fn() != nullptr;
}

int sm100_auto_splits(const mla_decode_args* a, int sms) {
  const int clusters = a->B * (a->H * a->Q / 128);
  const int pairs = sms / 2;
  const int tiles = (a->Lk + kTile - 1) / kTile;
  if (clusters >= pairs) return 1;
  int s = pairs / clusters;
  if (s > tiles) s = tiles;
  return s < 1 ? 1 : s;
}

cudaError_t launch_decode_sm100(const DecodeParams& p, const mla_decode_args* a, cudaStream_t st) {
  Sm100Params P;
  memset(&P, 0, sizeof(P));
  P.p = p;
  P.paged = a->block_table != nullptr;
  const uint64_t rows = (uint64_t)p.B * p.HQ;
  {
    uint64_t d[2] = {512, rows}, s[1] = {512 * 2};
    uint32_t box[2] = {64, 64};
    if (!encode_bf16(&P.tm_q, a->q_lat, 2, d, s, box)) return cudaErrorInvalidValue;
  }
  {
    uint64_t d[2] = {64, rows}, s[1] = {64 * 2};
    uint32_t box[2] = {64, 64};
    if (!encode_bf16(&P.tm_qpe, a->q_pe, 2, d, s, box)) return cudaErrorInvalidValue;
  }
  uint64_t rows_per = P.paged ? (uint64_t)a->page_size : (uint64_t)a->Lk;
  uint64_t outer = P.paged ? (uint64_t)a->num_pages : (uint64_t)a->B;
  uint64_t kv_outer_stride = P.paged ? (uint64_t)a->page_size * a->kv_row_stride * 2
                                     : (uint64_t)a->kv_batch_stride * 2;
  uint64_t pe_outer_stride = P.paged ? (uint64_t)a->page_size * a->pe_row_stride * 2
                                     : (uint64_t)a->pe_batch_stride * 2;
  if (!P.paged && a->B == 1) {
    kv_outer_stride = (uint64_t)a->Lk * a->kv_row_stride * 2;
    pe_outer_stride = (uint64_t)a->Lk * a->pe_row_stride * 2;
  }
  {
    // (64 dims, rows, 8 chunks of 64 dims, seq|page): a box of 64 rows x 2 chunks
    // lands as [chunk][row][128 B], two K-major (or MN-major) SW128 blocks
    uint64_t d[4] = {64, rows_per, 8, outer};
    uint64_t s[3] = {(uint64_t)a->kv_row_stride * 2, 128, kv_outer_stride};
    uint32_t bk[4] = {64, 64, 2, 1}, bk3[4] = {64, 64, 3, 1};
    if (!encode_bf16(&P.tm_k, a->kv_cache, 4, d, s, bk)) return cudaErrorInvalidValue;
    if (!encode_bf16(&P.tm_k3, a->kv_cache, 4, d, s, bk3)) return cudaErrorInvalidValue;
  }
  {
    uint64_t d[3] = {64, rows_per, outer};
    uint64_t s[2] = {(uint64_t)a->pe_row_stride * 2, pe_outer_stride};
    uint32_t bx[3] = {64, 64, 1};
    if (!encode_bf16(&P.tm_pe, a->pe_cache, 3, d, s, bx)) return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(decode_sm100_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (p.HQ / 128), p.B, p.num_splits);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, decode_sm100_kernel, P);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mla
