// block_bwd_internal.h -- launchers of the gate and adaLN backward
// (block_bwd.cu). Not part of the public ABI (that is include/mf.h).
#pragma once

#include <cstdint>

#include <cuda_runtime_api.h>

#include "mf_internal.h"

namespace mf {

// d_o = gate * dy; dmod[:, :, gate, :] = per-(sample, modality) sums of dy * O.
cudaError_t launch_gated_residual_bwd(const mf_bf16* dy, const mf_bf16* o, const float* mod,
                                      const int32_t* tok_sample, const uint8_t* tok_mod,
                                      int32_t T, int32_t S, int32_t hid, mf_bf16* d_o,
                                      float* dmod, const KernelCtl& ctl, cudaStream_t st);

// dx = resid + LayerNorm backward of dx_mod * (1 + scale); dmod[:, :, shift and
// scale, :] = per-(sample, modality) sums of dx_mod and dx_mod * xhat. stats:
// [T] (mean, rstd) pairs of workspace.
cudaError_t launch_adaln_modulate_bwd(const mf_bf16* dx_mod, const mf_bf16* x, const float* mod,
                                      const int32_t* tok_sample, const uint8_t* tok_mod,
                                      const mf_bf16* resid, int32_t T, int32_t S, int32_t hid,
                                      float eps, mf_bf16* dx, float* dmod, float* stats,
                                      const KernelCtl& ctl, cudaStream_t st);

// Backward of mod = c W: dW = c^T dmod ([C][6 hid]) and dc = dmod W^T ([S][C]);
// either output may be NULL.
cudaError_t launch_adaln_params_bwd(const float* dmod, const float* c, const float* W,
                                    int32_t S, int32_t C, int32_t hid, float* dc, float* dW,
                                    cudaStream_t st);

}  // namespace mf
