// vae_internal.h -- launchers of the Mage-VAE conv block's kernels (vae.cu).
// Not part of the public ABI (that is include/mf.h).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime_api.h>

#include "mf_internal.h"

namespace mf {

// GroupNorm statistics are folded per pixel chunk, then per (sample, group).
int gn_chunks(int32_t N, int32_t H, int32_t W);
size_t gn_workspace_bytes(int32_t N, int32_t H, int32_t W, int32_t G);

// y = SiLU(GroupNorm(x; gamma, beta)) on NHWC bf16; workspace of
// gn_workspace_bytes (partials, then per-group (mean, rstd)), 256-byte aligned.
cudaError_t launch_group_norm_silu(const mf_bf16* x, const float* gamma, const float* beta,
                                   int32_t N, int32_t H, int32_t W, int32_t C, int32_t G,
                                   float eps, mf_bf16* y, void* workspace, cudaStream_t st);

// The 128-pixel block (BH x BW) the conv tiles an H x W image with.
void conv_pixel_tile(int32_t H, int32_t W, int32_t* BH, int32_t* BW);

// y = conv3x3(x; Wt) + bias + residual on NHWC bf16 (bias / residual may be NULL);
// `pair`: on clusters of two CTAs (M = 256 MMAs over two vertically adjacent
// pixel tiles).
cudaError_t launch_conv3x3(const mf_bf16* x, const mf_bf16* Wt, const float* bias,
                           const mf_bf16* residual, int32_t N, int32_t H, int32_t W, int32_t Cin,
                           int32_t Cout, mf_bf16* y, bool pair, const KernelCtl& ctl,
                           cudaStream_t st);

}  // namespace mf
