// attn_bwd_internal.h -- launchers of the attention backward (attn_bwd.cu).
// Not part of the public ABI (that is include/mf.h).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime_api.h>

#include "mf_internal.h"

namespace mf {

// 128-row query tiles of a pack, each sample's tiles starting at its first
// token (the row tables of the backward are laid out per such tile).
int32_t bwd_query_tiles(const int32_t* cu_h, int32_t S);

// Workspace carve-up of the backward (all fp32, 256-byte aligned pieces):
// dq_acc [T][H][D], lse_tab and delta_tab [H][tiles][128].
size_t attn_bwd_workspace_bytes(int32_t T, int32_t S, int32_t H, int32_t D);

// Runs the three kernels of the backward on `st`: row tables + zeroing of the
// dQ accumulator, the tensor-core pass over (sample, head, key tile), and the
// dQ conversion to bf16.
cudaError_t launch_attention_bwd(const mf_bf16* q, const mf_bf16* k, const mf_bf16* v,
                                 const mf_bf16* o, const mf_bf16* d_o, const float* lse,
                                 const int32_t* cu_seqlens_d, const int32_t* cu_seqlens_h,
                                 int32_t S, int32_t T, int32_t H, int32_t D, float softmax_scale,
                                 mf_bf16* dq, mf_bf16* dk, mf_bf16* dv, void* workspace,
                                 const KernelCtl& ctl, cudaStream_t st);

}  // namespace mf
