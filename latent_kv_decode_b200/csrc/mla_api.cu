// C ABI of libmla (declared in include/mla.h): host-side validation, split
// selection, workspace layout and kernel dispatch. Nothing here allocates
// device memory or synchronises; every call enqueues on the caller's stream.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "append.h"
#include "common.cuh"
#include "launch.h"

namespace {

thread_local int g_last_cuda_error = 0;

mla_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MLA_OK;
  g_last_cuda_error = (int)e;
  return MLA_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
      n = v;
  }
  return n;
}

constexpr int kMaxSplits = 256;

bool dims_ok(int B, int H, int Q, int Dn, int Vd, int Ckv) {
  return B >= 1 && H >= 8 && H <= 128 && H % 8 == 0 && Q >= 1 && Q <= 4 &&
         (Dn == 64 || Dn == 128) && Vd == 128 && Ckv == mla::kCkv;
}

mla_status_t check_proj(const void* a, const void* w, const void* o, int B, int H, int Q, int Dn,
                        int Vd, int Ckv, mla_dtype_t dt) {
  if (!a || !w || !o) return MLA_ERR_INVALID_ARG;
  if (!aligned(a, 16) || !aligned(w, 16) || !aligned(o, 16)) return MLA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Q <= 0 || Dn <= 0 || Vd <= 0 || Ckv <= 0) return MLA_ERR_INVALID_ARG;
  if (dt != MLA_F32 && dt != MLA_BF16) return MLA_ERR_UNSUPPORTED;
  if (!dims_ok(B, H, Q, Dn, Vd, Ckv)) return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

// Which kernel family serves a decode call.
enum class DecodePath { kSimt, kSm100, kSm100Fp4 };

DecodePath pick_path(const mla_decode_args* a) {
  if (a->cache_dtype == MLA_FP4_E2M1_E4M3x16)
    return mla::sm100_fp4_decode_supported(a) ? DecodePath::kSm100Fp4 : DecodePath::kSimt;
  return mla::sm100_decode_supported(a) ? DecodePath::kSm100 : DecodePath::kSimt;
}

mla_status_t validate_decode(const mla_decode_args* a) {
  if (!a) return MLA_ERR_INVALID_ARG;
  if (a->B <= 0 || a->H <= 0 || a->Q <= 0 || a->Lk <= 0) return MLA_ERR_INVALID_ARG;
  if (a->q_dtype != MLA_F32 && a->q_dtype != MLA_BF16) return MLA_ERR_UNSUPPORTED;
  const bool fp4 = a->cache_dtype == MLA_FP4_E2M1_E4M3x16;
  if (!fp4 && a->cache_dtype != a->q_dtype) return MLA_ERR_UNSUPPORTED;
  if (fp4 && (a->q_dtype != MLA_BF16 || a->Dr != 0)) return MLA_ERR_UNSUPPORTED;
  if (a->Ckv != mla::kCkv) return MLA_ERR_UNSUPPORTED;
  if (!(a->Dr == 0 || a->Dr == 32 || a->Dr == 64)) return MLA_ERR_UNSUPPORTED;
  if (a->H < 8 || a->H > 128 || a->H % 8 != 0 || a->Q > 4) return MLA_ERR_UNSUPPORTED;
  if (a->rope_tail != 0 && a->rope_tail != 64) return MLA_ERR_UNSUPPORTED;
  if (a->num_splits < 0 || a->num_splits > kMaxSplits) return MLA_ERR_INVALID_ARG;
  if (!a->q_lat || !a->kv_cache || !a->x) return MLA_ERR_INVALID_ARG;
  if (a->Dr > 0 && (!a->q_pe || !a->pe_cache)) return MLA_ERR_INVALID_ARG;
  if (!aligned(a->q_lat, 16) || !aligned(a->kv_cache, 16) || !aligned(a->x, 16))
    return MLA_ERR_INVALID_ARG;
  if (a->Dr > 0 && (!aligned(a->q_pe, 16) || !aligned(a->pe_cache, 16)))
    return MLA_ERR_INVALID_ARG;
  if ((a->lse && !aligned(a->lse, 4)) || (a->sinks && !aligned(a->sinks, 4)) ||
      (a->seq_lens && !aligned(a->seq_lens, 4)) ||
      (a->block_table && !aligned(a->block_table, 4)) || (a->err_flag && !aligned(a->err_flag, 4)))
    return MLA_ERR_INVALID_ARG;
  const int64_t esz = a->q_dtype == MLA_F32 ? 4 : 2;
  if (fp4) {
    if (a->kv_row_stride < mla::kFp4EntryBytes || a->kv_row_stride % 16 != 0)
      return MLA_ERR_INVALID_ARG;
  } else {
    if (a->kv_row_stride < a->Ckv || (a->kv_row_stride * esz) % 16 != 0)
      return MLA_ERR_INVALID_ARG;
    if (a->Dr > 0 && (a->pe_row_stride < a->Dr || (a->pe_row_stride * esz) % 16 != 0))
      return MLA_ERR_INVALID_ARG;
  }
  if (a->block_table) {
    if (a->page_size <= 0 || a->max_pages <= 0 || a->num_pages <= 0) return MLA_ERR_INVALID_ARG;
    if ((int64_t)a->max_pages * a->page_size < a->Lk) return MLA_ERR_INVALID_ARG;
  } else {
    if (a->kv_batch_stride < (int64_t)a->Lk * a->kv_row_stride && a->B > 1)
      return MLA_ERR_INVALID_ARG;
    if (a->Dr > 0 && a->pe_batch_stride < (int64_t)a->Lk * a->pe_row_stride && a->B > 1)
      return MLA_ERR_INVALID_ARG;
  }
  if (!(a->softmax_scale > 0.f) || !isfinite(a->softmax_scale)) return MLA_ERR_INVALID_ARG;
  if (a->rope_tail && !(a->rope_theta > 0.f)) return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

int resolve_splits(const mla_decode_args* a) {
  if (a->num_splits > 0) return a->num_splits;
  const int tiles = (a->Lk + mla::kTile - 1) / mla::kTile;
  if (pick_path(a) == DecodePath::kSm100) return mla::sm100_auto_splits(a, sm_count());
  if (pick_path(a) == DecodePath::kSm100Fp4) return mla::sm100_fp4_auto_splits(a, sm_count());
  // generic path: about two CTAs of 16 rows per SM
  const int ctas = a->B * ((a->H * a->Q + 15) / 16);
  int s = (2 * sm_count() + ctas - 1) / ctas;
  s = s < 1 ? 1 : s;
  s = s > tiles ? tiles : s;
  s = s > 64 ? 64 : s;
  return s;
}

size_t ws_bytes(const mla_decode_args* a, int S) {
  if (S <= 1) return 0;
  const size_t rows = (size_t)S * a->B * a->H * a->Q;
  size_t o = rows * a->Ckv * sizeof(float);
  o = (o + 255) & ~(size_t)255;
  return o + rows * sizeof(float);
}

mla::DecodeParams make_params(const mla_decode_args* a, int S, void* ws) {
  mla::DecodeParams p;
  memset(&p, 0, sizeof(p));
  p.B = a->B;
  p.H = a->H;
  p.Q = a->Q;
  p.HQ = a->H * a->Q;
  p.Ckv = a->Ckv;
  p.Dr = a->Dr;
  p.D = a->Ckv + a->Dr;
  p.q_lat = a->q_lat;
  p.q_pe = a->q_pe;
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
  p.mask = a->causal_mask;
  p.causal = a->causal;
  p.scale = a->softmax_scale;
  p.scale_log2 = a->softmax_scale * 1.4426950408889634f;
  p.sinks = a->sinks;
  p.rope_tail = a->rope_tail;
  p.rope_theta = a->rope_theta;
  p.num_splits = S;
  p.x = a->x;
  p.lse = a->lse;
  p.err = a->err_flag;
  if (S > 1 && ws) {
    const size_t rows = (size_t)S * a->B * a->H * a->Q;
    size_t o = rows * a->Ckv * sizeof(float);
    o = (o + 255) & ~(size_t)255;
    p.ws_o = (float*)ws;
    p.ws_lse = (float*)((char*)ws + o);
  }
  return p;
}

}  // namespace

extern "C" {

const char* mla_status_string(mla_status_t s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
  }
  return "MLA_ERR_UNKNOWN";
}

int mla_last_cuda_error(void) { return g_last_cuda_error; }

const char* mla_version(void) { return "0.1.0"; }

mla_status_t mla_absorb_q(const void* q_nope, const void* wkv_b, void* q_lat, int B, int H, int Q,
                          int Dn, int Vd, int Ckv, mla_dtype_t dt, void* stream) {
  mla_status_t s = check_proj(q_nope, wkv_b, q_lat, B, H, Q, Dn, Vd, Ckv, dt);
  if (s != MLA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if (dt == MLA_BF16 && mla::sm100_proj_supported(B, H, Q, Dn, Vd, Ckv, q_nope, wkv_b, q_lat))
    return cuda_status(mla::launch_absorb_sm100(q_nope, wkv_b, q_lat, B, H, Q, Dn, Vd, Ckv, st));
  return cuda_status(
      mla::launch_absorb_simt(q_nope, wkv_b, q_lat, B, H, Q, Dn, Vd, Ckv, dt == MLA_BF16, st));
}

mla_status_t mla_up_proj(const void* x, const void* wkv_b, void* out, int B, int H, int Q, int Dn,
                         int Vd, int Ckv, mla_dtype_t dt, void* stream) {
  mla_status_t s = check_proj(x, wkv_b, out, B, H, Q, Dn, Vd, Ckv, dt);
  if (s != MLA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if (dt == MLA_BF16 && mla::sm100_proj_supported(B, H, Q, Dn, Vd, Ckv, x, wkv_b, out))
    return cuda_status(mla::launch_up_proj_sm100(x, wkv_b, out, B, H, Q, Dn, Vd, Ckv, st));
  return cuda_status(
      mla::launch_up_proj_simt(x, wkv_b, out, B, H, Q, Dn, Vd, Ckv, dt == MLA_BF16, st));
}

int mla_decode_num_splits(const mla_decode_args* a) {
  if (validate_decode(a) != MLA_OK) return -1;
  return resolve_splits(a);
}

size_t mla_decode_workspace_size(const mla_decode_args* a) {
  if (validate_decode(a) != MLA_OK) return 0;
  return ws_bytes(a, resolve_splits(a));
}

mla_status_t mla_decode(const mla_decode_args* a, void* workspace, size_t workspace_bytes,
                        void* stream) {
  mla_status_t s = validate_decode(a);
  if (s != MLA_OK) return s;
  const int S = resolve_splits(a);
  const size_t need = ws_bytes(a, S);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 256)))
    return MLA_ERR_WORKSPACE;
  mla::DecodeParams p = make_params(a, S, workspace);
  cudaStream_t st = (cudaStream_t)stream;
  const DecodePath path = pick_path(a);
  if (path == DecodePath::kSm100) return cuda_status(mla::launch_decode_sm100(p, a, st));
  if (path == DecodePath::kSm100Fp4) return cuda_status(mla::launch_decode_fp4_sm100(p, a, st));
  return cuda_status(mla::launch_decode_simt(p, a->q_dtype == MLA_BF16,
                                             a->cache_dtype == MLA_FP4_E2M1_E4M3x16, st));
}

mla_status_t mla_combine(const mla_decode_args* a, const void* workspace, size_t workspace_bytes,
                         void* stream) {
  mla_status_t s = validate_decode(a);
  if (s != MLA_OK) return s;
  const int S = resolve_splits(a);
  if (S <= 1) return MLA_OK;
  const size_t need = ws_bytes(a, S);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return MLA_ERR_WORKSPACE;
  mla::DecodeParams p = make_params(a, S, (void*)workspace);
  return cuda_status(mla::launch_combine_simt(p, a->q_dtype == MLA_BF16, (cudaStream_t)stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without any device allocation: the split-KV partials live in a
// library-owned array in device memory instead of a caller workspace.
// ---------------------------------------------------------------------------

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_static_scratch[MLA_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_static_scratch_mu;
void* g_static_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device. Host code only
// sees a host-side stand-in for the array, so the address is looked up once
// per device, with that device current, and cached.
mla_status_t static_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (!g_static_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_status(e);
    g_static_scratch_ptr[dev] = p;
  }
  *out = g_static_scratch_ptr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" mla_status_t mla_decode_static_scratch(const mla_decode_args* a, void* stream) {
  mla_status_t s = validate_decode(a);
  if (s != MLA_OK) return s;
  const size_t need = ws_bytes(a, resolve_splits(a));
  if (need > (size_t)MLA_STATIC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE;
  void* ws = nullptr;
  if (need > 0) {
    s = static_scratch_address(&ws);
    if (s != MLA_OK) return s;
  }
  s = mla_decode(a, ws, need, stream);
  if (s != MLA_OK) return s;
  return mla_combine(a, ws, need, stream);
}

// ---------------------------------------------------------------------------
// cache append
// ---------------------------------------------------------------------------
namespace {

mla_status_t validate_append(const mla_append_args* a) {
  if (!a) return MLA_ERR_INVALID_ARG;
  if (a->B <= 0 || a->Q <= 0 || a->Lk <= 0 || a->Ckv <= 0 || a->Dr < 0) return MLA_ERR_INVALID_ARG;
  if (a->src_dtype != MLA_F32 && a->src_dtype != MLA_BF16) return MLA_ERR_UNSUPPORTED;
  const bool fp4 = a->cache_dtype == MLA_FP4_E2M1_E4M3x16;
  if (!fp4 && a->cache_dtype != a->src_dtype) return MLA_ERR_UNSUPPORTED;
  if (!a->c_kv || !a->kv_cache || !a->seq_lens) return MLA_ERR_INVALID_ARG;
  if (a->Dr > 0 && (!a->k_pe || !a->pe_cache)) return MLA_ERR_INVALID_ARG;
  if (!aligned(a->seq_lens, 4) || (a->block_table && !aligned(a->block_table, 4)) ||
      (a->err_flag && !aligned(a->err_flag, 4)))
    return MLA_ERR_INVALID_ARG;
  const int64_t esz = a->src_dtype == MLA_F32 ? 4 : 2;
  if (!aligned(a->c_kv, esz) || (a->Dr > 0 && !aligned(a->k_pe, esz))) return MLA_ERR_INVALID_ARG;
  if (fp4) {
    if (a->Ckv != mla::kCkv || a->Dr != 0) return MLA_ERR_UNSUPPORTED;
    if (a->rope_tail != 0 && a->rope_tail != 64) return MLA_ERR_UNSUPPORTED;
    if (a->rope_tail && !(a->rope_theta > 0.f)) return MLA_ERR_INVALID_ARG;
    // 8-byte code stores: entries start on 16-byte boundaries
    if (!aligned(a->kv_cache, 16) || a->kv_row_stride < mla::kFp4EntryBytes || a->kv_row_stride % 16 != 0)
      return MLA_ERR_INVALID_ARG;
    if (!a->block_table && a->kv_batch_stride % 16 != 0) return MLA_ERR_INVALID_ARG;
  } else {
    if (a->rope_tail != 0) return MLA_ERR_UNSUPPORTED;   // rope rows arrive rotated
    if (!aligned(a->kv_cache, esz) || a->kv_row_stride < a->Ckv) return MLA_ERR_INVALID_ARG;
    if (a->Dr > 0 && (!aligned(a->pe_cache, esz) || a->pe_row_stride < a->Dr)) return MLA_ERR_INVALID_ARG;
  }
  if (a->block_table) {
    if (a->page_size <= 0 || a->max_pages <= 0 || a->num_pages <= 0) return MLA_ERR_INVALID_ARG;
    if ((int64_t)a->max_pages * a->page_size < a->Lk) return MLA_ERR_INVALID_ARG;
  } else if (a->B > 1) {
    if (a->kv_batch_stride < (int64_t)a->Lk * a->kv_row_stride) return MLA_ERR_INVALID_ARG;
    if (a->Dr > 0 && a->pe_batch_stride < (int64_t)a->Lk * a->pe_row_stride) return MLA_ERR_INVALID_ARG;
  }
  return MLA_OK;
}

}  // namespace

extern "C" mla_status_t mla_cache_append(const mla_append_args* a, void* stream) {
  mla_status_t s = validate_append(a);
  if (s != MLA_OK) return s;
  return cuda_status(mla::launch_cache_append(a, (cudaStream_t)stream));
}

namespace {

bool is_sm100() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10;
}

mla_status_t validate_group_wo(const mla_group_wo_args* a) {
  if (!a) return MLA_ERR_INVALID_ARG;
  if (a->B <= 0 || a->H <= 0 || a->Q <= 0 || a->Ckv <= 0 || a->G <= 0 || a->R <= 0)
    return MLA_ERR_INVALID_ARG;
  if (a->wo_b && a->D <= 0) return MLA_ERR_INVALID_ARG;
  if (!a->x || !a->wo_a || !a->out) return MLA_ERR_INVALID_ARG;
  if (!aligned(a->x, 16) || !aligned(a->wo_a, 16) || !aligned(a->out, 16) || !aligned(a->wo_b, 16))
    return MLA_ERR_INVALID_ARG;
  if (a->dtype != MLA_BF16) return MLA_ERR_UNSUPPORTED;
  if (a->H % a->G != 0 || a->Ckv % 64 != 0 || a->R % 128 != 0 || a->Q > 16) return MLA_ERR_UNSUPPORTED;
  if (a->wo_b && a->D % 128 != 0) return MLA_ERR_UNSUPPORTED;
  // the TMA views index rows with 32-bit coordinates
  if ((int64_t)a->B * a->H * a->Q * a->Ckv >= ((int64_t)1 << 31)) return MLA_ERR_UNSUPPORTED;
  if ((int64_t)a->G * a->R * (a->H / a->G) * a->Ckv >= ((int64_t)1 << 31)) return MLA_ERR_UNSUPPORTED;
  if (!is_sm100()) return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

}  // namespace

extern "C" size_t mla_group_wo_workspace_size(const mla_group_wo_args* a) {
  if (validate_group_wo(a) != MLA_OK) return 0;
  return mla::group_wo_workspace_bytes(a, sm_count());
}

extern "C" mla_status_t mla_group_wo(const mla_group_wo_args* a, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  mla_status_t s = validate_group_wo(a);
  if (s != MLA_OK) return s;
  const size_t need = mla::group_wo_workspace_bytes(a, sm_count());
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 256))) return MLA_ERR_WORKSPACE;
  return cuda_status(mla::launch_group_wo_sm100(a, workspace, sm_count(), (cudaStream_t)stream));
}
