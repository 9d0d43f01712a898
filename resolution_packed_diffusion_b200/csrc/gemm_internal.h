// gemm_internal.h -- launch interface of the modality-specific linear layer,
// shared by the library's translation units. Not part of the public ABI (that
// is include/mf.h).
#pragma once

#include <cstdint>

#include <cuda_runtime_api.h>

#include "mf.h"

namespace mf {

struct KernelCtl;

// Jobs of the modality-specific linear layer: one per (128-row tile, modality
// present in it); job = tile | modality << 15.
constexpr int kMaxGemmTiles = 1024;  // packs of up to 131072 tokens
struct GemmJobs {
  int32_t n;
  uint16_t job[2 * kMaxGemmTiles];
};

// Fills the job list from each sample's image and text token counts (image
// tokens first in a sample); false if the pack has too many tiles.
bool build_gemm_jobs(const int32_t* n_img, const int32_t* n_txt, int32_t S, int32_t T,
                     GemmJobs* jobs);

cudaError_t launch_modality_linear(const mf_bf16* x, const mf_bf16* W, const uint8_t* tok_mod,
                                   const GemmJobs& jobs, int32_t T, int32_t K, int32_t N,
                                   int32_t act, mf_bf16* out, const KernelCtl& ctl,
                                   cudaStream_t st);

}  // namespace mf
