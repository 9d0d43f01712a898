// gemm_internal.h -- launch interface of the modality-specific linear layer,
// shared by the library's translation units. Not part of the public ABI (that
// is include/mf.h).
#pragma once

#include <cstdint>

#include <cuda_runtime_api.h>

#include "mf.h"

namespace mf {

struct KernelCtl;

// Jobs of the modality-specific linear layer: one per (row block, modality
// present in it); job = block | modality << 15. A row block is 128 rows for the
// one-CTA kernel and 256 for the CTA-pair kernel (gemm_job_rows).
constexpr int kMaxGemmTiles = 1024;  // packs of up to 131072 tokens
struct GemmJobs {
  int32_t n;
  uint16_t job[2 * kMaxGemmTiles];
};

// Rows of a job: 128, or 256 with CTA pairs.
int gemm_job_rows(bool pair);

// The linear-layer kernel form chosen for the current device
// (mf_set_linear_cta_pair, mf_api.cu); false if the device cannot be read.
bool linear_cta_pair(bool* pair);

// Fills the job list from each sample's image and text token counts (image
// tokens first in a sample) for row blocks of `rows` (gemm_job_rows); false if
// the pack has too many blocks or `rows` is not a job size.
bool build_gemm_jobs(const int32_t* n_img, const int32_t* n_txt, int32_t S, int32_t T,
                     int32_t rows, GemmJobs* jobs);

// `pair`: run on clusters of two CTAs (jobs built for gemm_job_rows(true)).
cudaError_t launch_modality_linear(const mf_bf16* x, const mf_bf16* W, const uint8_t* tok_mod,
                                   const GemmJobs& jobs, bool pair, int32_t T, int32_t K,
                                   int32_t N, int32_t act, mf_bf16* out, const KernelCtl& ctl,
                                   cudaStream_t st);

// out[t] = x[t] W^T for every row t < T with one weight matrix W [N][K] (no
// modality split, no activation): the weight-gradient and transposed products
// of the backward.
cudaError_t launch_linear_plain(const mf_bf16* x, const mf_bf16* W, int32_t T, int32_t K,
                                int32_t N, bool pair, mf_bf16* out, const KernelCtl& ctl,
                                cudaStream_t st);

}  // namespace mf
