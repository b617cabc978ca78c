/*
 * mla.h - C ABI of libmla.so: single-step Multi-Head Latent Attention decode
 * with weight absorption, on NVIDIA B200 (sm_100a).
 *
 * The operation is mla_decode_step of the 6547.cn exam question "MLA 单步解码":
 *
 *   q_lat  = q_nope . W_UK[h]                      (blank [1])   mla_absorb_q
 *   logit  = (q_lat . kv[t] + q_pe . pe[t]) * scale (blanks [2],[3])
 *   logit  = -inf where t is not visible           (blank [4])
 *   x      = softmax(logit) . kv                   (step 5)      mla_decode
 *                                                                 (+ mla_combine)
 *   out    = x . W_UV[h]^T                         (blank [5])   mla_up_proj
 *
 * with wkv_b (H, Dn+Vd, Ckv) split as W_UK = rows [0,Dn), W_UV = the last Vd
 * rows (the question's weight-split lines). The absorbed score
 * q_absorbed . c_kv + q_rope . k_rope is the associativity step written in
 * the comments of MultiHeadLatentAttention.forward_inference on the neuronix
 * page "DeepSeek-V3/R1 架构深度全景解析". The shared-latent variant (K = V =
 * one 512-dim latent stored as FP4 E2M1 with an E4M3 scale per 16 channels,
 * a sink logit per head, inverse RoPE on the output's last 64 dims) is the
 * openarchlab DeepSeek-V4.1-Flash page "4A · Multi-head Latent Attention"
 * (§1 Định nghĩa, §2 Luồng, §4 Profiling); the grouped output projection that
 * follows it there (§2 Luồng, §3 W_O nhóm) is mla_group_wo. The step before
 * the decode, writing a new token into its cache slot, is mla_cache_append.
 *
 * Conventions for every call:
 *  - Tensor pointers are DEVICE pointers owned by the caller. The library
 *    allocates no device memory and keeps no per-call state; calls are
 *    re-entrant. The one piece of library-global device state is the scratch
 *    array of mla_decode_static_scratch (a static device array, with its
 *    address looked up once per device); no other call touches it. Arrays
 *    are row-major (C order) and densely packed unless a stride argument says
 *    otherwise.
 *  - Every call only enqueues work on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and returns without synchronising.
 *  - Arguments are validated on the host before anything is enqueued; a call
 *    that returns anything but MLA_OK has enqueued nothing, except
 *    MLA_ERR_CUDA, which reports a failed launch (see mla_last_cuda_error).
 *  - Device pointers must be 16-byte aligned.
 *  - Supported shapes (decode, projections, combine, append): Ckv = 512; Dr
 *    in {0 (shared-latent variant), 32, 64}; Dn in {64, 128}; Vd = 128; H a
 *    multiple of 8, at most 128; Q in [1, 4]. mla_group_wo states its own.
 *    Anything else returns MLA_ERR_UNSUPPORTED.
 */
#ifndef LATENT_KV_DECODE_MLA_H
#define LATENT_KV_DECODE_MLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mla_status {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,  /* null/shape/stride/alignment/range error */
  MLA_ERR_UNSUPPORTED = 2,  /* dims or dtype combination not built */
  MLA_ERR_WORKSPACE = 3,    /* workspace missing or too small */
  MLA_ERR_CUDA = 4          /* a launch failed; mla_last_cuda_error() has the code */
} mla_status_t;

typedef enum mla_dtype {
  MLA_F32 = 0,              /* IEEE float32 */
  MLA_BF16 = 1,             /* bfloat16 storage, float32 arithmetic */
  MLA_FP4_E2M1_E4M3x16 = 2  /* cache only: 288-byte entries, see mla_decode_args */
} mla_dtype_t;

/* Human-readable name of a status code (static string, never NULL). */
const char* mla_status_string(mla_status_t s);

/* cudaError_t of the last MLA_ERR_CUDA returned on the calling host thread (0 if none). */
int mla_last_cuda_error(void);

/* Library version, e.g. "0.1.0". */
const char* mla_version(void);

/*
 * mla_absorb_q - blank [1] of mla_decode_step: q_lat[b,h,q,:] = q_nope[b,h,q,:] . W_UK[h].
 *
 *   q_nope (B,H,Q,Dn)      dtype dt
 *   wkv_b  (H,Dn+Vd,Ckv)   dtype dt; rows [0,Dn) of each head are W_UK[h]
 *   q_lat  (B,H,Q,Ckv)     dtype dt, written
 * dt is MLA_F32 or MLA_BF16; accumulation is float32.
 */
mla_status_t mla_absorb_q(const void* q_nope, const void* wkv_b, void* q_lat, int B, int H,
                          int Q, int Dn, int Vd, int Ckv, mla_dtype_t dt, void* stream);

/*
 * mla_up_proj - blank [5] of mla_decode_step: out[b,h,q,:] = W_UV[h] . x[b,h,q,:].
 *
 *   x      (B,H,Q,Ckv)     dtype dt
 *   wkv_b  (H,Dn+Vd,Ckv)   dtype dt; the last Vd rows of each head are W_UV[h]
 *   out    (B,H,Q,Vd)      dtype dt, written
 */
mla_status_t mla_up_proj(const void* x, const void* wkv_b, void* out, int B, int H, int Q,
                         int Dn, int Vd, int Ckv, mla_dtype_t dt, void* stream);

/*
 * Arguments of mla_decode / mla_combine: blanks [2]-[4] and step 5 of
 * mla_decode_step over a compressed cache, with optional ragged lengths,
 * paging, causal speculative queries, sinks and split-KV.
 *
 * Query (rows r = (b, h, q)):
 *   q_lat   (B,H,Q,Ckv) dtype q_dtype. For the shared-latent variant this is the
 *           query itself (already RoPE-rotated on its tail).
 *   q_pe    (B,H,Q,Dr)  dtype q_dtype, or NULL when Dr == 0.
 *
 * Cache (cache_dtype = q_dtype, or MLA_FP4_E2M1_E4M3x16 with Dr == 0):
 *   Contiguous (block_table == NULL): token t of sequence b is row
 *     kv_cache + b*kv_batch_stride + t*kv_row_stride (in elements), and the
 *     same with pe_* for pe_cache; the question's kv_cache (B,Lk,Ckv) and
 *     pe_cache (B,Lk,Dr) have row strides Ckv and Dr. A combined 576-wide
 *     row (latent then rope) is kv_cache = base, pe_cache = base + 512, both
 *     row strides 576.
 *   Paged (block_table != NULL): kv_cache/pe_cache point at pools of
 *     num_pages pages of page_size rows; token t of sequence b is row
 *     (block_table[b*max_pages + t/page_size]*page_size + t%page_size) of the
 *     pool, with the given row strides (batch strides unused).
 *   FP4: each row is one 288-byte entry (strides in BYTES): bytes 0..255 hold
 *     512 E2M1 codes, channel 2i in the low nibble of byte i and 2i+1 in the
 *     high nibble; bytes 256..287 hold the E4M3 scale of channels 16g..16g+15.
 *     K = V = the dequantised latent (openarchlab 4A §1, 288 B per entry).
 *
 * Visibility of token t to row (b,h,q): t < len_b (len_b = seq_lens[b], or Lk
 *   when seq_lens is NULL) and causal_mask[t] != 0 (when causal_mask is given;
 *   the question's (1,1,1,Lk) mask, 1 = visible) and, when `causal` is
 *   non-zero, t <= len_b - Q + q (the Q new tokens are the last Q rows).
 *   A row that sees nothing gets x = 0 and lse = -inf.
 *
 * Softmax: logit = score * softmax_scale. With `sinks` (H floats) the
 *   denominator also holds exp(sinks[h]) (a raw logit, not scaled), which
 *   carries no value (openarchlab 4A §2 attn_sink column).
 * Epilogue: rope_tail in {0, 64}: x's last rope_tail dims are rotated back by
 *   the query position len_b - Q + q, pairs (D-tail+2j, D-tail+2j+1) by angle
 *   -pos * rope_theta^(-2j/tail) (openarchlab 4A §2 inverse RoPE).
 *
 * Outputs: x (B,H,Q,Ckv) in q_dtype; lse (B,H,Q) float32 natural-log softmax
 *   denominator (tokens and sink), or NULL.
 *
 * Split-KV: num_splits = 0 picks a count from the SM count and the shape
 *   (mla_decode_num_splits reports it). With 1 split, mla_decode writes x and
 *   lse itself. With S > 1 splits, sequence b's tokens are cut into S ranges
 *   of whole 64-token tiles; mla_decode writes each range's normalised
 *   partial output and log-sum-exp into the workspace, and mla_combine must
 *   then be called with the same arguments and workspace to write x and lse.
 *
 * err_flag: optional device int32; the kernels OR in MLA_DEVICE_ERR_* bits
 *   when they meet bad data (a block_table entry outside [0,num_pages)) and
 *   skip that data instead of reading out of bounds. The caller clears it.
 */
typedef struct mla_decode_args {
  int B, H, Q;
  int Ckv;                 /* 512 */
  int Dr;                  /* 0, 32 or 64 */
  mla_dtype_t q_dtype;     /* MLA_F32 or MLA_BF16 (q_lat, q_pe, x) */
  mla_dtype_t cache_dtype; /* q_dtype, or MLA_FP4_E2M1_E4M3x16 */
  const void* q_lat;
  const void* q_pe;
  const void* kv_cache;
  const void* pe_cache;
  int64_t kv_row_stride, pe_row_stride;      /* elements (bytes for FP4) */
  int64_t kv_batch_stride, pe_batch_stride;  /* contiguous layout only */
  int Lk;                  /* contiguous: rows per sequence; paged: max_pages*page_size */
  const int32_t* seq_lens; /* (B) or NULL */
  const int32_t* block_table; /* (B,max_pages) or NULL */
  int max_pages, page_size, num_pages;
  const uint8_t* causal_mask; /* (Lk) or NULL */
  int causal;
  float softmax_scale;
  const float* sinks;      /* (H) or NULL */
  int rope_tail;           /* 0 or 64 */
  float rope_theta;
  int num_splits;          /* 0 = auto */
  void* x;                 /* out (B,H,Q,Ckv) */
  float* lse;              /* out (B,H,Q) or NULL */
  int32_t* err_flag;       /* optional device status word */
} mla_decode_args;

#define MLA_DEVICE_ERR_BLOCK_TABLE 1  /* a page id outside [0,num_pages) or a seq_lens entry outside [0,Lk] */
#define MLA_DEVICE_ERR_TIMEOUT 2      /* a bounded wait inside a kernel gave up */

/* Resolved split count for these arguments (>= 1), or -1 if they are invalid. */
int mla_decode_num_splits(const mla_decode_args* a);

/* Workspace bytes mla_decode needs for these arguments (0 when 1 split). */
size_t mla_decode_workspace_size(const mla_decode_args* a);

/*
 * mla_decode - scores against the compressed cache, mask, softmax and latent
 * aggregation (blanks [2]-[4] and step 5). `workspace` is a device buffer of
 * at least mla_decode_workspace_size(a) bytes (may be NULL when that is 0).
 */
mla_status_t mla_decode(const mla_decode_args* a, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * mla_combine - merge the split partials that mla_decode left in `workspace`:
 * L = log(sum_s e^{lse_s} [+ e^{sink_h}]), x = sum_s e^{lse_s - L} O_s, then
 * the inverse-RoPE epilogue; writes a->x and a->lse. A no-op returning MLA_OK
 * when the resolved split count is 1.
 */
mla_status_t mla_combine(const mla_decode_args* a, const void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * mla_decode_static_scratch - mla_decode followed by mla_combine, for callers
 * that may not allocate device memory. The source pages have no counterpart: this is
 * a deployment variant of the two calls above.
 *
 * Some callers cannot call cudaMalloc or take memory from an allocator: a
 * serving engine that reserved nearly all of HBM for its KV cache at start-up
 * (an allocation at decode time would fail), or a plugin hook of a host
 * runtime that forbids allocation inside the hook. This entry point needs no
 * workspace argument: the split-KV partials go to one array of
 * MLA_STATIC_SCRATCH_BYTES bytes of device memory that the library owns,
 * which every GPU that loads the library holds until the process exits.
 *
 *   - Takes the same arguments as mla_decode and writes a->x and a->lse; they
 *     are final when the work it enqueued on `stream` completes.
 *   - Returns MLA_ERR_WORKSPACE, enqueuing nothing, when the resolved split
 *     count needs more than MLA_STATIC_SCRATCH_BYTES (see
 *     mla_decode_workspace_size); one split needs no scratch at all.
 *   - The first call on each device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *     The address is kept for the life of the process, so this entry point
 *     does not support cudaDeviceReset (which reloads the module and moves
 *     the array) between its calls on a device.
 *   - All calls share the one array, whatever the stream. Calls whose GPU
 *     work overlaps in time race on it and give wrong results: serialise them
 *     (one stream, or events). The array keeps the last call's contents;
 *     nothing in it needs to start at zero, because mla_decode writes every
 *     partial that mla_combine reads in the same call.
 *   - Calls no cudaMalloc, cudaFree or allocating library routine.
 */
#define MLA_STATIC_SCRATCH_BYTES (32u << 20)
mla_status_t mla_decode_static_scratch(const mla_decode_args* a, void* stream);

/*
 * mla_cache_append - the step before the decode: write each sequence's Q new
 * tokens into the cache rows mla_decode reads. The neuronix DeepSeek-V3/R1
 * page's LatentKVCachePool gives a token's latent and rope parts a slot at its
 * position before attention runs; the openarchlab 4A page (§1, §4) stores the
 * shared latent, its tail rotated at the token's position, as a 288-byte FP4
 * entry.
 *
 *   c_kv  (B,Q,Ckv) new latent rows, src_dtype, contiguous.
 *   k_pe  (B,Q,Dr)  new rope rows (already rotated), src_dtype, contiguous;
 *         NULL when Dr == 0.
 *   seq_lens (B) int32, required: the lengths AFTER the append. New token i
 *     of sequence b is token t = seq_lens[b] - Q + i and goes to the row that
 *     mla_decode reads for t: the same kv_cache / pe_cache, row and batch
 *     strides, Lk, block_table, max_pages, page_size and num_pages rules.
 *   cache_dtype == src_dtype (MLA_F32 or MLA_BF16): the rows are copied.
 *   cache_dtype == MLA_FP4_E2M1_E4M3x16 (Ckv = 512, Dr = 0, src MLA_F32 or
 *     MLA_BF16, row stride in BYTES, >= 288 and a multiple of 16): the
 *     latent's last rope_tail (0 or 64) dims are rotated by +t, pairs
 *     (448+2j, 449+2j) by angle t * rope_theta^(-2j/64) (angles in double,
 *     results rounded to float); then each group of 16 channels gets
 *     scale = E4M3(amax / 6) and codes E2M1(x / scale), both rounded to
 *     nearest-even from float32 quotients with saturation (x's sign kept; a
 *     zero scale gives zero codes), in the entry layout mla_decode reads.
 *   err_flag: optional device int32; a token with t outside [0, Lk) or a page
 *     id outside [0, num_pages) sets MLA_DEVICE_ERR_BLOCK_TABLE and is not
 *     written.
 */
typedef struct mla_append_args {
  int B, Q;
  int Ckv, Dr;
  mla_dtype_t src_dtype;   /* MLA_F32 or MLA_BF16 (c_kv, k_pe) */
  mla_dtype_t cache_dtype; /* src_dtype, or MLA_FP4_E2M1_E4M3x16 */
  const void* c_kv;
  const void* k_pe;
  void* kv_cache;
  void* pe_cache;
  int64_t kv_row_stride, pe_row_stride;      /* elements (bytes for FP4) */
  int64_t kv_batch_stride, pe_batch_stride;  /* contiguous layout only */
  int Lk;                  /* contiguous: rows per sequence; paged: max_pages*page_size */
  const int32_t* seq_lens; /* (B), lengths after the append */
  const int32_t* block_table; /* (B,max_pages) or NULL */
  int max_pages, page_size, num_pages;
  int rope_tail;           /* FP4 only: 0 or 64 */
  float rope_theta;
  int32_t* err_flag;       /* optional device status word */
} mla_append_args;

mla_status_t mla_cache_append(const mla_append_args* a, void* stream);

/*
 * mla_group_wo - the step after the shared-latent decode's inverse RoPE: the
 * grouped low-rank output projection (openarchlab DeepSeek-V4.1-Flash 4A,
 * §2 Luồng "Group-LoRA W_O (8 nhóm × 1024)" back to [B, T, D_model]; §3 W_O
 * nhóm: each group of heads has its own small projection, the groups'
 * results side by side).
 *
 * For every token t = b*Q + q and group g of the G groups of H/G
 * consecutive heads:
 *   u_g[t]          = x[b, g*H/G .. (g+1)*H/G - 1, q, :] laid head-major ((H/G)*Ckv values)
 *   z[t, g*R + r]   = sum_k wo_a[g, r, k] * u_g[t, k]           (group g's own factor)
 *   out[t, n]       = sum_k wo_b[n, k] * z[t, k]                 (shared factor; omitted
 *                                                                 when wo_b is NULL: out = z)
 * D_model is not given by the page; D is the caller's.
 *
 * Layouts (row-major, bf16, device pointers owned by the caller, 16-byte
 * aligned): x (B,H,Q,Ckv); wo_a (G,R,(H/G)*Ckv); wo_b (D,G*R) or NULL;
 * out (B,Q,D), or (B,Q,G*R) without wo_b.
 * Supported: q/weight dtype MLA_BF16, Ckv a multiple of 64, H a multiple of
 *   G, R and D multiples of 128, Q in 1..16; fp32 accumulation, z rounded
 *   to bf16 between the two factors. Anything else: MLA_ERR_UNSUPPORTED.
 * workspace: at least mla_group_wo_workspace_size(a) bytes of device memory
 *   (z and the split-K partial sums), or NULL when that is 0; smaller gives
 *   MLA_ERR_WORKSPACE with nothing enqueued.
 * err_flag: optional device int32; MLA_DEVICE_ERR_TIMEOUT when a bounded
 *   wait inside the kernel gave up (the output is then not written).
 */
typedef struct mla_group_wo_args {
  int B, H, Q, Ckv;
  int G, R, D;             /* groups, rank per group, output width (ignored without wo_b) */
  mla_dtype_t dtype;       /* MLA_BF16 */
  const void* x;
  const void* wo_a;
  const void* wo_b;        /* or NULL */
  void* out;
  int32_t* err_flag;       /* optional device status word */
} mla_group_wo_args;

size_t mla_group_wo_workspace_size(const mla_group_wo_args* a);
mla_status_t mla_group_wo(const mla_group_wo_args* a, void* workspace, size_t workspace_bytes,
                          void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LATENT_KV_DECODE_MLA_H */
