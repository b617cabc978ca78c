// Tensor-core decode for bf16 caches (Ckv = 512, Dr = 64, H*Q a multiple of
// 128): blanks [2]-[4] and step 5 of mla_decode_step (the 6547.cn MLA decode
// question), with the absorbed score of the neuronix DeepSeek-V3/R1 page.
//
// One 2-CTA cluster per (128-row block, sequence, split). Per 128-token tile
// of the cache, CTA r loads its own 64 tokens [64r, 64r+64) once: the eight
// 64-dim latent chunks as two 32 KB TMA boxes (chunks 0, 1, 4, 5 into slots
// 0-3 and chunks 2, 3, 6, 7 into slots 4-7 of the tile's set) and the rope
// chunk.
//
//   S  = Q . K^T       pair MMA, M = 128 (CTA r: query rows [64r, 64r+64)),
//                      N = the 128 tokens (each CTA supplies its 64), K = 576.
//   softmax            online, base 2, lazy rescale (a row's running max only
//                      moves when a score exceeds it by more than 2^8).
//   O^T += V^T . P^T   pair MMA, M = 256 latent dims (CTA r: dims
//                      [256n + 128r, +128) for n = 0, 1), N = the 128 query
//                      rows (each CTA supplies its rows' P), K = the tokens.
//
// Accumulating O transposed puts 128 rows of the tensor datapath on every
// SM for the aggregation (the latent dims), where O = P . V would give each
// SM only its 64 query rows. The price: for its dims, CTA r needs the peer's
// 64 tokens too. After S(j) is computed, the four latent chunks CTA r does
// not aggregate are dead in its shared memory; the peer tokens' chunks of
// CTA r's dims are loaded from L2 (the peer just brought them in from HBM)
// into exactly those slots, which is where the pair MMA's A descriptor finds
// "tokens of the other CTA" in both CTAs. Every cache row crosses HBM once.
//
// With that slot order, slots 2n, 2n+1 hold the dims of O^T half n that CTA 0
// aggregates and slots 4 + 2n, 5 + 2n those of CTA 1; the tokens of CTA 0
// (the first four 16-token MMA steps of the aggregation) are read from slots
// 0-3 in both CTAs and those of CTA 1 from slots 4-7. Each CTA's peer-token
// data is one 32 KB box into the four slots holding the dims it does not
// aggregate, and the aggregation is issued as two halves (slots 0-3, then
// slots 4-7) so the next tile's first box can load as soon as the first half
// is done. Only two tile sets fit beside Q in shared memory.
//
// A row's rescale factor alpha touches O^T in both CTAs (column = row), so
// each CTA sends its rows' alpha (and whether any row needs a rescale) to the
// peer every tile; the rescale itself is rare.
//
// Warp roles (384 threads): warp 0 own-token producer (+ Q), warp 1 QK issuer
// (even CTA) and TMEM owner, warps 2-5 and 8-11 softmax + epilogue (TMEM lane
// = 32*(warp%4) + lane; the two sets split each lane's 64 scores), warp 6
// peer-token producer, warp 7 PV issuer (even CTA). The two issuers write disjoint TMEM (S and O^T) and each commit
// tracks only its own thread's MMAs, so neither stream waits on the other's
// barriers. Every wait is bounded; a timeout sets MLA_DEVICE_ERR_TIMEOUT and
// the kernel unwinds.
#include <cudaTypedefs.h>
#include <math.h>

#include "common.cuh"
#include "launch.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kThreads = 384;
constexpr int kTileT = 128;                 // tokens per tile (both CTAs)
constexpr int kChunk = 8192;                // 64 rows (tokens or query rows) x 128 B
constexpr int kQBytes = 9 * kChunk;         // q_lat chunks 0-7, q_pe

constexpr int kOffQ = 0;
constexpr int kOffL = kOffQ + kQBytes;      // 2 sets x 8 latent chunk slots
constexpr int kOffR = kOffL + 16 * kChunk;  // rope chunk slot
constexpr int kOffP = kOffR + kChunk;       // P: 2 blocks (tokens 0-63, 64-127) of 64 rows x 128 B
constexpr int kBigBytes = kOffP + 2 * kChunk;   // the 1024-aligned operand region
enum : int {
  B_QFULL = 0,
  B_KF0 = 1,              // [2] latent chunks 0-3 of both CTAs landed
  B_KF1 = 3,              // [2] latent chunks 2, 3, 6, 7 (slots 4-7) of both CTAs landed
  B_XF = 5,               // [2] peer-token chunks of both CTAs landed
  B_SFULL = 7,            // [2] S(j) computed (both CTAs, multicast commit)
  B_SFREE = 9,            // [2] S buffer read by both CTAs (count 2)
  B_PFULL = 11,           // P(j) written and O^T rescaled by both CTAs (count 2)
  B_PVDONE = 12,          // [2] O^T += V^T P^T of tile j done (both CTAs, multicast)
  B_AX = 14,              // [2] the peer's alpha of tile j arrived (64 + 1 asynchronous 4-byte stores)
  B_EPX = 16,             // the peer's output scales arrived (64 asynchronous 4-byte stores)
  B_QH0 = 17,             // [2] QK(j) over slots 0-3 done (both CTAs, multicast)
  B_PVX = 19,             // [2] PV(j) over slots 0-3 done (both CTAs, multicast)
  B_RF = 21,              // the rope chunk of tile j of both CTAs landed (phase j)
  B_RFREE = 22,           // QK(j) over the rope chunk done: the rope slot is free (multicast)
  B_COUNT = 23
};
// Control block (barriers, TMEM address, abort flag, rescale flags): in the
// alignment gap below the operand region when it fits there, else after the
// exchange block. Exchange block (row statistics, alpha): after the operands.
constexpr int kOffTmemPtr = 8 * B_COUNT;                  // within the control block
constexpr int kOffAbort = kOffTmemPtr + 4;
constexpr int kOffFlags = kOffAbort + 4;                  // int need[2][2]
constexpr int kCtrlBytes = (kOffFlags + 16 + 15) & ~15;
constexpr int kOffXmax = kBigBytes;                       // float [2 sets][128 lanes]
constexpr int kOffAlpha = kOffXmax + 1024;                // float [2][128]: alpha (epilogue: output scale)
constexpr int kXchgEnd = kOffAlpha + 1024;
constexpr int kSmemAlloc = 232448;                        // the per-block limit
// the base is 16-byte aligned: a gap below kCtrlBytes leaves the control
// block after the exchange block, a larger one (at most 1008) holds it
static_assert(kXchgEnd + kCtrlBytes + (kCtrlBytes - 16) <= kSmemAlloc, "shared memory over the per-block limit");
static_assert(kXchgEnd + 1008 <= kSmemAlloc, "shared memory over the per-block limit");

constexpr uint32_t kColS = 0;               // S buffers at columns 0 and 64 (pair M = 128 layout)
constexpr uint32_t kColO = 128;             // O^T halves n = 0, 1 at columns 128 and 256
constexpr uint32_t kTmemCols = 512;

constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

struct alignas(64) Sm100Params {
  CUtensorMap tm_q;    // q_lat  (B*HQ, 512), box 64 x 64
  CUtensorMap tm_qpe;  // q_pe   (B*HQ, 64),  box 64 x 64
  CUtensorMap tm_kx;   // latent cache as (64 dims, rows, 4 chunks, 2 groups of 4, seq|page):
                       // box 64 rows x 2 chunks x 2 groups = chunks c, c+1, c+4, c+5
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
  const uint32_t ctrl = (sb0 - raw >= (uint32_t)kCtrlBytes) ? raw : sb0 + kXchgEnd;
  uint8_t* ctrl_p = smem_raw + (ctrl - raw);
  const DecodeParams& p = P.p;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int rb = blockIdx.x >> 1, b = blockIdx.y, z = blockIdx.z;
  pdl_launch_dependents();
  auto bar = [&](int i) -> uint32_t { return ctrl + 8u * (uint32_t)i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl_p + kOffAbort);

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_KF0 + i), 1);
      mbar_init(bar(B_KF1 + i), 1);
      mbar_init(bar(B_XF + i), 1);
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_SFREE + i), 2);   // one arrival per CTA
      mbar_init(bar(B_PVDONE + i), 1);
      mbar_init(bar(B_AX + i), 1);      // local expect_tx; the peer's stores count the bytes
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_QH0 + i), 1);
      mbar_init(bar(B_PVX + i), 1);
    }
    mbar_init(bar(B_RF), 1);
    mbar_init(bar(B_RFREE), 1);
    mbar_init(bar(B_PFULL), 2);         // one arrival per CTA
    mbar_init(bar(B_EPX), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_2sm(ctrl + kOffTmemPtr, kTmemCols);
    tmem_relinquish_2sm();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(ctrl_p + kOffTmemPtr);
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
  // TMA coordinates of the 64 tokens starting at t: (row, seq|page)
  auto coords = [&](int t, int& y, int& zc) {
    if (P.paged) {
      zc = page_of(p, b, t, len);
      y = 0;
    } else {
      zc = b;
      y = t;
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ own-token producer
    if (lane == 0) {
      tma_prefetch_desc(&P.tm_q);
      tma_prefetch_desc(&P.tm_qpe);
      tma_prefetch_desc(&P.tm_kx);
      tma_prefetch_desc(&P.tm_pe);
      const int qrow = b * p.HQ + rb * 128 + (int)rank * 64;
      const uint32_t qbar = map_to_rank(bar(B_QFULL), 0);
      if (rank == 0) mbar_arrive_expect_tx(bar(B_QFULL), 2 * kQBytes);
      for (int c = 0; c < 8; ++c) tma_load_2d_2sm(sb0 + kOffQ + c * kChunk, &P.tm_q, qbar, 64 * c, qrow);
      tma_load_2d_2sm(sb0 + kOffQ + 8 * kChunk, &P.tm_qpe, qbar, 0, qrow);
      // L2 prefetch of this CTA's 64 cache rows of tile jt (latent and rope rows
      // as contiguous ranges), one tile ahead of its shared-memory load: the
      // load in the tile-to-tile dependency chain then hits L2
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
        // each range ends at the last row's own data (strided rows may share a buffer)
        prefetch_l2_bulk(kvb, (uint32_t)(((int64_t)(rows - 1) * p.kv_row + p.Ckv) * 2));
        prefetch_l2_bulk(peb, (uint32_t)(((int64_t)(rows - 1) * p.pe_row + p.Dr) * 2));
      };
      bool ok = true;
      for (int j = 0; j < ntiles && ok; ++j) {
        const int s = j & 1;
        prefetch_tile(j + 1);
        int y, zc;
        coords(t_begin + j * kTileT + (int)rank * 64, y, zc);
        // the single rope slot once QK(j-1) has read it (QK takes the rope chunk
        // first, so this load runs a latent box ahead of the tile's own boxes)
        if (j >= 1 && !mbar_wait_cluster(bar(B_RFREE), (j - 1) & 1)) { ok = false; break; }
        if (rank == 0) mbar_arrive_expect_tx(bar(B_RF), 2 * kChunk);
        tma_load_3d_2sm(sb0 + kOffR, &P.tm_pe, map_to_rank(bar(B_RF), 0), 0, y, zc);
        // slots 0-3 of set s held tile j-2 until the first half of its aggregation
        if (j >= 2 && !mbar_wait_cluster(bar(B_PVX + s), ((j - 2) >> 1) & 1)) { ok = false; break; }
        const uint32_t dst = sb0 + kOffL + s * 8 * kChunk;
        if (rank == 0) mbar_arrive_expect_tx(bar(B_KF0 + s), 2 * 4 * kChunk);
        tma_load_5d_2sm(dst, &P.tm_kx, map_to_rank(bar(B_KF0 + s), 0), 0, y, 0, 0, zc);
        // slots 4-7 until the second half
        if (j >= 2 && !mbar_wait_cluster(bar(B_PVDONE + s), ((j - 2) >> 1) & 1)) { ok = false; break; }
        if (rank == 0) mbar_arrive_expect_tx(bar(B_KF1 + s), 2 * 4 * kChunk);
        tma_load_5d_2sm(dst + 4 * kChunk, &P.tm_kx, map_to_rank(bar(B_KF1 + s), 0), 0, y, 2, 0, zc);
        if (*abort_flag) ok = false;
      }
      if (!ok) {
        fail();
        settle();
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    // ------------------------------------------------------------------ peer-token producer
    // The peer tokens' chunks of this CTA's aggregation dims (CTA 0: chunks 0,
    // 1, 4, 5; CTA 1: 2, 3, 6, 7) go, as one box, to the four slots holding the
    // chunks this CTA does not aggregate (CTA 0: slots 4-7, free once S(j) is
    // computed; CTA 1: slots 0-3, free once QK(j) has passed them).
    if (lane == 0) {
      bool ok = true;
      for (int j = 0; j < ntiles && ok; ++j) {
        const int s = j & 1;
        if (!mbar_wait_cluster(bar((rank == 0 ? B_SFULL : B_QH0) + s), (j >> 1) & 1)) { ok = false; break; }
        int y, zc;
        coords(t_begin + j * kTileT + (1 - (int)rank) * 64, y, zc);
        if (rank == 0) mbar_arrive_expect_tx(bar(B_XF + s), 2 * 4 * kChunk);
        tma_load_5d_2sm(sb0 + kOffL + (s * 8 + 4 * (1 - (int)rank)) * kChunk, &P.tm_kx,
                        map_to_rank(bar(B_XF + s), 0), 0, y, 2 * (int)rank, 0, zc);
        if (*abort_flag) ok = false;
      }
      if (!ok) {
        fail();
        settle();
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ QK issuer (even CTA)
    // S(j) = Q . K^T in three groups as their data lands: the rope chunk (then
    // a commit that frees the rope slot for tile j+1), slots 0-3 (then a commit
    // that frees them for the peer-token box of CTA 1), slots 4-7; the S buffer
    // must have been read by softmax(j-2).
    if (rank == 0 && lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      const uint64_t qd0 = smem_desc(sb0 + kOffQ, 16, 1024, kSwizzle128B);
      const uint64_t kd0 = smem_desc(sb0 + kOffL, 16, 1024, kSwizzle128B);
      const uint64_t rd0 = smem_desc(sb0 + kOffR, 16, 1024, kSwizzle128B);
      bool ok = mbar_wait_cluster(bar(B_QFULL), 0);
      for (int j = 0; j < ntiles && ok; ++j) {
        const int s = j & 1;
        const uint32_t d = tmem + kColS + 64u * s;
        if (j >= 2) ok = mbar_wait_cluster(bar(B_SFREE + s), ((j - 2) >> 1) & 1);
#pragma unroll 1
        for (int g3 = 0; g3 < 3 && ok; ++g3) {
          ok = g3 == 0 ? mbar_wait_cluster(bar(B_RF), j & 1)
                       : mbar_wait_cluster(bar((g3 == 1 ? B_KF0 : B_KF1) + s), (j >> 1) & 1);
          if (!ok) break;
          tc_fence_after();
          const int nc = g3 == 0 ? 1 : 4;
#pragma unroll 1
          for (int cc = 0; cc < nc; ++cc) {
            // the rope, then slot 4 (g3 - 1) + cc holding latent chunk (0, 1, 4, 5, 2, 3, 6, 7)[slot]
            const int slot = 4 * (g3 - 1) + cc;
            const int c = g3 == 0 ? 8 : ((slot & 2) << 1) | ((slot & 4) >> 1) | (slot & 1);
            const uint64_t qd = desc_advance(qd0, c * kChunk);
            const uint64_t kd = g3 == 0 ? rd0 : desc_advance(kd0, (s * 8 + slot) * kChunk);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_bf16_ss_2sm(d, desc_advance(qd, 32 * k), desc_advance(kd, 32 * k), idesc_qk,
                              (g3 | cc | k) != 0);
          }
          if (g3 == 0) mma_commit_2sm_mc(bar(B_RFREE), 3);
          if (g3 == 1) mma_commit_2sm_mc(bar(B_QH0 + s), 3);
        }
        if (ok) mma_commit_2sm_mc(bar(B_SFULL + s), 3);
        if (*abort_flag) ok = false;
      }
      if (!ok) fail();
    }
    __syncwarp();
  } else if (warp == 7) {
    // ------------------------------------------------------------------ PV issuer (even CTA)
    // O^T += V^T . P^T once P(j) is written by both CTAs and the peer tokens
    // are in: first the tokens of CTA 0 (slots 2n, 2n+1 for O^T half n), a
    // commit that frees slots 0-3, then the tokens of CTA 1 (slots 4+2n, 5+2n).
    if (rank == 0 && lane == 0) {
      const uint32_t idesc_pv = idesc_bf16_f32(256, 128, true, false);
      const uint64_t vd0 = smem_desc(sb0 + kOffL, kChunk, 1024, kSwizzle128B);
      const uint64_t pd0 = smem_desc(sb0 + kOffP, 16, 1024, kSwizzle128B);
      bool ok = true;
      for (int j = 0; j < ntiles && ok; ++j) {
        const int s = j & 1;
        ok = mbar_wait_cluster(bar(B_PFULL), j & 1) && mbar_wait_cluster(bar(B_XF + s), (j >> 1) & 1);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int hv = 0; hv < 2; ++hv) {
#pragma unroll
          for (int n = 0; n < 2; ++n) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t vd = desc_advance(vd0, (s * 8 + 4 * hv + 2 * n) * kChunk + kk * 2048);
              const uint64_t pd = desc_advance(pd0, hv * kChunk + kk * 32);
              mma_bf16_ss_2sm(tmem + kColO + 128u * n, vd, pd, idesc_pv,
                              (j > 0 || hv > 0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit_2sm_mc(bar((hv == 0 ? B_PVX : B_PVDONE) + s), 3);
        }
        if (*abort_flag) ok = false;
      }
      if (!ok) fail();
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    // Two warp sets read each TMEM lane quarter: set 0 (warps 2-5) takes the
    // first 32 of the lane's 64 tokens, set 1 (warps 8-11) the last 32, so a
    // query row's scores sit with four threads (two token halves x two sets).
    const int g = warp & 3;
    const int sset = warp >= 8 ? 1 : 0;
    const int L = 32 * g + lane;                // TMEM lane
    const int half = L >> 6, row = L & 63;      // S: this CTA's query row, token half
    const int xi = 128 * sset + L;              // this thread's slot in the row-statistics exchange
    const bool owner = half == 0 && sset == 0;  // one thread per query row sends its stats
    const int r = rb * 128 + (int)rank * 64 + row;
    const int q = r % p.Q;
    const int h = r / p.Q;
    const uint32_t lane_base = (uint32_t)(32 * g) << 16;
    float* xmax = reinterpret_cast<float*>(smem + kOffXmax);
    float* alpha_s = reinterpret_cast<float*>(smem + kOffAlpha);
    int* need_s = reinterpret_cast<int*>(ctrl_p + kOffFlags);
    const uint32_t peer = rank ^ 1u;
    float m_run = -INFINITY, l_part = 0.f;
    bool ab = false;
    // loop-invariant parameters, read once into registers
    const float sl2 = p.scale_log2;
    const uint8_t* mask = p.mask;
    const bool causal = p.causal != 0;
    const int causal_last = len - p.Q + q;   // last visible token of a causal row
    const bool paged = p.block_table != nullptr;
    const bool leader_thread = (xi == 0);    // arrives for this CTA on the even CTA's barriers

    for (int j = 0; j < ntiles; ++j) {
      const int sbuf = j & 1;
      float s[32];
      // this tile's alpha exchange: 64 rescale factors and one flag from the peer
      if (leader_thread) mbar_arrive_expect_tx(bar(B_AX + (j & 1)), 65 * 4);
      if (!ab) ab = !mbar_wait_cluster(bar(B_SFULL + sbuf), (j >> 1) & 1);
      ab = __any_sync(0xffffffffu, ab);
      if (!ab) {
        tc_fence_after();
        uint32_t v[2][16];
#pragma unroll
        for (int c = 0; c < 2; ++c) tmem_ld16(tmem + lane_base + kColS + 64u * sbuf + 32u * sset + 16u * c, v[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int i = 0; i < 16; ++i) s[16 * c + i] = __uint_as_float(v[c][i]);
      }
      tc_fence_before();

      // scale to log2 units and mask: this thread holds tokens [ts, ts + 32) of
      // the 64-token block (one page) at tb; tokens [ts, ts + lim) pass the
      // range / causal / page tests
      const int tb = t_begin + j * kTileT + 64 * half;
      const int ts = tb + 32 * sset;
      int lim = t_end - ts;
      if (causal) lim = min(lim, causal_last - ts + 1);
      if (paged && !page_ok(p, b, tb < len ? tb : 0)) lim = 0;
      if (ab) lim = 0;
      // four independent max chains (one warp per SM sub-partition: latency, not
      // throughput, sets the pace)
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (mask == nullptr) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          s[c] = (c < lim) ? s[c] * sl2 : -INFINITY;
          mx4[c & 3] = fmaxf(mx4[c & 3], s[c]);
        }
      } else {
        // the question's mask, one byte per lane (ts is the same across the warp)
        const uint32_t m0 = __ballot_sync(0xffffffffu, ts + lane < t_end && mask[ts + lane] != 0);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const bool vis = c < lim && ((m0 >> c) & 1u);
          s[c] = vis ? s[c] * sl2 : -INFINITY;
          mx4[c & 3] = fmaxf(mx4[c & 3], s[c]);
        }
      }
      float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      xmax[xi] = mx;
      // all eight warps have read S(j) by now: release the buffer to the MMA
      // (the arrival publishes no data; tcgen05.wait::ld already returned)
      const bool stop = bar_or(1, 256, ab);
      if (leader_thread) mbar_arrive_remote_relaxed(map_to_rank(bar(B_SFREE + sbuf), 0));
      if (stop) {
        ab = true;
        break;
      }
      mx = fmaxf(fmaxf(mx, xmax[xi ^ 64]), fmaxf(xmax[xi ^ 128], xmax[xi ^ 192]));
      const float m_new = fmaxf(m_run, mx);
      // the first visible score sets the reference (O^T is still zero then)
      const bool need = m_run != -INFINITY && (m_new - m_run) > kRescaleThreshold;
      float alpha = 1.f;
      if (need) alpha = exp2f(m_run - m_new);
      if (need || m_run == -INFINITY) m_run = m_new;
      uint32_t pk[16];
      float ps4[4] = {0.f, 0.f, 0.f, 0.f};
      const bool none = (m_run == -INFINITY);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float p0 = none ? 0.f : fast_exp2(s[2 * c] - m_run);
        const float p1 = none ? 0.f : fast_exp2(s[2 * c + 1] - m_run);
        ps4[c & 3] += p0 + p1;
        pk[c] = pack_bf16(p0, p1);
      }
      l_part = l_part * alpha + ((ps4[0] + ps4[1]) + (ps4[2] + ps4[3]));

      // this CTA's rows' alpha to both CTAs (O^T column = query row)
      const int abuf = j & 1;
      const int col = (int)rank * 64 + row;
      const uint32_t peer_ax = map_to_rank(bar(B_AX + abuf), peer);
      if (owner) {
        alpha_s[abuf * 128 + col] = alpha;
        st_async_b32(map_to_rank(smem_u32(alpha_s + abuf * 128 + col), peer), __float_as_uint(alpha), peer_ax);
      }
      const bool need_cta = bar_or(1, 256, owner && need);
      if (leader_thread) {
        st_async_b32(map_to_rank(smem_u32(need_s + abuf * 2 + (int)rank), peer), need_cta ? 1u : 0u, peer_ax);
      }

      // the P buffer (and O^T) are free once PV(j-1) is done
      if (j >= 1 && !ab) ab = !mbar_wait_cluster(bar(B_PVDONE + ((j - 1) & 1)), ((j - 1) >> 1) & 1);
      if (!ab) ab = !mbar_wait_cluster(bar(B_AX + abuf), (j >> 1) & 1);
      ab = __any_sync(0xffffffffu, ab);
      uint8_t* prow = smem + kOffP + half * kChunk + row * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 val = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow + 16 * ((4 * sset + c) ^ (row & 7))) = val;
      }
      // rescale O^T columns whose row's running max moved (either CTA's rows);
      // set n rescales O^T half n
      const bool rescale = !ab && j > 0 && (need_cta || need_s[abuf * 2 + (int)peer] != 0);
      if (rescale) {
        tc_fence_after();
        const float* al = alpha_s + abuf * 128;
        {
          const int n = sset;
#pragma unroll 1
          for (int c = 0; c < 128; c += 32) {
            uint32_t v[2][16];
            const uint32_t ta = tmem + lane_base + kColO + 128u * n + (uint32_t)c;
            tmem_ld16(ta, v[0]);
            tmem_ld16(ta + 16u, v[1]);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 2; ++k) {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                v[k][i] = __float_as_uint(__uint_as_float(v[k][i]) * al[c + 16 * k + i]);
              tmem_st16(ta + 16u * k, v[k]);
            }
          }
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      // P(j) of all eight warps is written: one arrival for this CTA
      named_bar_sync(2, 256);
      if (leader_thread) mbar_arrive_remote_cta(map_to_rank(bar(B_PFULL), 0));
    }

    // ---------------------------------------------------------------- epilogue
    // row statistics: both token halves, then each row's output scale to both CTAs
    ab = bar_or(1, 256, ab);
    xmax[xi] = l_part;
    named_bar_sync(2, 256);
    const float l_tot = (xmax[row] + xmax[64 + row]) + (xmax[128 + row] + xmax[192 + row]);
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
    // every row's output scale, in O^T column order, to both CTAs: into the
    // alpha buffer the last tile did not use (the peer may still be reading
    // that one for its last rescale)
    float* scl = alpha_s + (ntiles & 1) * 128;
    if (leader_thread) mbar_arrive_expect_tx(bar(B_EPX), 64 * 4);
    if (owner) {
      const int col = (int)rank * 64 + row;
      scl[col] = scale_o;
      st_async_b32(map_to_rank(smem_u32(scl + col), peer), __float_as_uint(scale_o),
                   map_to_rank(bar(B_EPX), peer));
    }
    const int64_t grow = (int64_t)b * p.HQ + r;
    if (owner) {
      if (p.num_splits > 1)
        p.ws_lse[(int64_t)z * p.B * p.HQ + grow] = lse;
      else if (p.lse)
        p.lse[grow] = lse;
    }
    if (ntiles > 0 && !ab) ab = !mbar_wait_cluster(bar(B_PVDONE + ((ntiles - 1) & 1)), ((ntiles - 1) >> 1) & 1);
    if (!ab) ab = !mbar_wait_cluster(bar(B_EPX), 0);
    ab = __any_sync(0xffffffffu, ab);
    ab = bar_or(1, 256, ab);
    if (ab) fail();
    tc_fence_after();
    const bool have_o = ntiles > 0 && !ab;
    // this thread's O^T lane is latent dim d of half n; its 128 columns are the
    // block's rows. Each warp (32 dims) moves 16 rows at a time through shared
    // memory (the free tile slots) so the output goes out as 16-byte stores of
    // whole 64- or 128-byte row pieces.
    const int64_t row0 = (int64_t)b * p.HQ + rb * 128;
    // inverse RoPE of the tail: dims (D - tail + 2i, D - tail + 2i + 1) sit in
    // lanes (L, L ^ 1); the rotation angle depends on the query index only
    const int tail0 = p.Ckv - p.rope_tail;
    const bool split = p.num_splits > 1;
    uint8_t* stage = smem + kOffL + (4 * sset + g) * 2048;   // 16 rows x 32 dims x 4 B per warp
    {
      const int n = sset;   // set n writes O^T half n
      const int d0 = 256 * n + 128 * (int)rank + 32 * g;   // this warp's first dim
      const int d = d0 + lane;
      const bool rot = !split && p.rope_tail > 0 && d0 + 31 >= tail0;
      // cos / sin of the rotation for query index 0..3 (Q <= 4)
      float c0v = 1.f, c1v = 1.f, c2v = 1.f, c3v = 1.f, s0v = 0.f, s1v = 0.f, s2v = 0.f, s3v = 0.f;
      if (rot && d >= tail0) {
        const double freq = pow((double)p.rope_theta, -2.0 * (double)((d - tail0) >> 1) / (double)p.rope_tail);
        double sd, cd;
        sincos(-(double)(len - p.Q) * freq, &sd, &cd);
        c0v = (float)cd;
        s0v = (float)sd;
        if (p.Q > 1) {
          sincos(-(double)(len - p.Q + 1) * freq, &sd, &cd);
          c1v = (float)cd;
          s1v = (float)sd;
        }
        if (p.Q > 2) {
          sincos(-(double)(len - p.Q + 2) * freq, &sd, &cd);
          c2v = (float)cd;
          s2v = (float)sd;
        }
        if (p.Q > 3) {
          sincos(-(double)(len - p.Q + 3) * freq, &sd, &cd);
          c3v = (float)cd;
          s3v = (float)sd;
        }
      }
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 16) {
        uint32_t v[16];
        if (have_o) {
          tmem_ld16(tmem + lane_base + kColO + 128u * n + (uint32_t)c0, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = 0u;
        }
        float f[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) f[i] = __uint_as_float(v[i]) * scl[c0 + i];
        if (rot) {
          // the partner lane holds the other element of the pair
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float o = __shfl_xor_sync(0xffffffffu, f[i], 1);
            if (d >= tail0) {
              const int qq = (rb * 128 + c0 + i) % p.Q;
              const float cc = qq == 0 ? c0v : qq == 1 ? c1v : qq == 2 ? c2v : c3v;
              const float ss = qq == 0 ? s0v : qq == 1 ? s1v : qq == 2 ? s2v : s3v;
              f[i] = (L & 1) ? (o * ss + f[i] * cc) : (f[i] * cc - o * ss);
            }
          }
        }
        if (split) {
          // fp32 partials: [16 rows][32 dims] = 128 B per row, 4 x 16 B per lane
          float* st = reinterpret_cast<float*>(stage);
#pragma unroll
          for (int i = 0; i < 16; ++i) st[i * 32 + lane] = f[i];
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int rr = (lane >> 3) + 4 * k, ch = lane & 7;
            const uint4 val = *reinterpret_cast<const uint4*>(st + rr * 32 + 4 * ch);
            *reinterpret_cast<uint4*>(p.ws_o + ((int64_t)z * p.B * p.HQ + row0 + c0 + rr) * p.Ckv + d0 + 4 * ch) = val;
          }
        } else {
          // bf16 output: [16 rows][32 dims] = 64 B per row, 2 x 16 B per lane
          __nv_bfloat16* st = reinterpret_cast<__nv_bfloat16*>(stage);
#pragma unroll
          for (int i = 0; i < 16; ++i) st[i * 32 + lane] = __float2bfloat16_rn(f[i]);
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int rr = (lane >> 2) + 8 * k, ch = lane & 3;
            const uint4 val = *reinterpret_cast<const uint4*>(st + rr * 32 + 8 * ch);
            *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.x) + (row0 + c0 + rr) * p.Ckv + d0 + 8 * ch) = val;
          }
        }
        __syncwarp();
      }
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
  cuuint32_t elem[5] = {1, 1, 1, 1, 1};
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
    // (64 dims, rows, 4 chunks, 2 groups of 4 chunks, seq|page): a box of 64 rows
    // x 2 chunks x 2 groups lands as four K-major SW128 blocks of 8 KB, chunks
    // (c, c+1, c+4, c+5) for a start chunk c of 0 or 2
    uint64_t d[5] = {64, rows_per, 4, 2, outer};
    uint64_t s[4] = {(uint64_t)a->kv_row_stride * 2, 128, 512, kv_outer_stride};
    uint32_t bx[5] = {64, 64, 2, 2, 1};
    if (!encode_bf16(&P.tm_kx, a->kv_cache, 5, d, s, bx)) return cudaErrorInvalidValue;
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
