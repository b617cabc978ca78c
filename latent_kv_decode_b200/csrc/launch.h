// Host-side launchers of libmla's kernels (internal; the public ABI is include/mla.h).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace mla {

cudaError_t launch_absorb_simt(const void* q_nope, const void* wkv_b, void* q_lat, int B, int H,
                               int Q, int Dn, int Vd, int Ckv, bool bf16, cudaStream_t st);
cudaError_t launch_up_proj_simt(const void* x, const void* wkv_b, void* out, int B, int H, int Q,
                                int Dn, int Vd, int Ckv, bool bf16, cudaStream_t st);
size_t decode_simt_smem(int D);
cudaError_t launch_decode_simt(const DecodeParams& p, bool bf16, bool fp4, cudaStream_t st);
cudaError_t launch_combine_simt(const DecodeParams& p, bool bf16, cudaStream_t st);

// tensor-core per-head projections (bf16): Ckv = 512, Vd = 128, Dn in {64, 128}, 16-byte
// aligned activation, weight and output pointers
bool sm100_proj_supported(int B, int H, int Q, int Dn, int Vd, int Ckv, const void* act,
                          const void* w, const void* out);
cudaError_t launch_absorb_sm100(const void* q_nope, const void* wkv_b, void* q_lat, int B, int H,
                                int Q, int Dn, int Vd, int Ckv, cudaStream_t st);
cudaError_t launch_up_proj_sm100(const void* x, const void* wkv_b, void* out, int B, int H, int Q,
                                 int Dn, int Vd, int Ckv, cudaStream_t st);

// tensor-core (tcgen05, 1-SM, M = 64) decode for the shared-latent FP4 cache: bf16 q,
// Ckv = 512, Dr = 0, H*Q % 64 == 0, contiguous 288-byte entries (row stride 288)
bool sm100_fp4_decode_supported(const mla_decode_args* a);
int sm100_fp4_auto_splits(const mla_decode_args* a, int sms);
cudaError_t launch_decode_fp4_sm100(const DecodeParams& p, const mla_decode_args* a, cudaStream_t st);

// tensor-core (tcgen05, 2-CTA cluster) decode for bf16, Ckv=512, Dr=64, H*Q % 128 == 0
bool sm100_decode_supported(const mla_decode_args* a);
int sm100_auto_splits(const mla_decode_args* a, int sms);
cudaError_t launch_decode_sm100(const DecodeParams& p, const mla_decode_args* a, cudaStream_t st);

// grouped low-rank output projection (tcgen05 weight-streaming GEMM with split-K):
// bf16, Ckv % 64 == 0, H % G == 0, R and D multiples of 128, Q <= 16
size_t group_wo_workspace_bytes(const mla_group_wo_args* a, int sms);
cudaError_t launch_group_wo_sm100(const mla_group_wo_args* a, void* ws, int sms, cudaStream_t st);

}  // namespace mla
