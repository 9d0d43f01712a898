// mf_internal.h -- declarations shared by the library's translation units.
// Not part of the public ABI (that is include/mf.h).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime_api.h>

#include "mf.h"

namespace mf {

// Passed by value to every kernel: where to record a device-side failure and
// how long any single wait may last.
struct KernelCtl {
  int* err;
  uint64_t wait_limit_ns;
};

// Per-device error word and wait limit (mf_api.cu).
cudaError_t get_ctl(KernelCtl* ctl);

// Host offsets of a pack: true when 0 = cu_h[0] <= cu_h[1] <= ... <= cu_h[S]
// <= MF_MAX_TOKENS; then *T = cu_h[S].
bool check_offsets(const int32_t* cu_h, int32_t S, int32_t* T);

// Descriptor data of a pack, passed by value to the id kernel.
struct PackParams {
  int32_t S;
  int32_t T;
  int32_t cu[MF_MAX_SAMPLES + 1];
  int32_t frames[MF_MAX_SAMPLES];
  int32_t grid_h[MF_MAX_SAMPLES];
  int32_t grid_w[MF_MAX_SAMPLES];
};

// RoPE tables computed on the host in double precision: inverse frequency and
// driving position component (0 f, 1 h, 2 w; -1 = unrotated) of every pair.
struct RopeTable {
  float inv_freq[64];
  int32_t comp[64];
};
void make_rope_table(int32_t D, int32_t rope_axes, float base, RopeTable* tab);

// Launchers (each returns the launch's cudaError_t).
cudaError_t launch_pack_ids(const PackParams& p, int32_t* cu_d, int32_t* pos_ids,
                            int32_t* tok_sample, uint8_t* tok_mod, cudaStream_t st);
cudaError_t launch_adaln_params(const float* c, const float* W, int32_t S, int32_t C,
                                int32_t hid, float* mod, cudaStream_t st);
cudaError_t launch_adaln_modulate(const mf_bf16* x, const float* mod, const int32_t* tok_sample,
                                  const uint8_t* tok_mod, int32_t T, int32_t S, int32_t hid,
                                  float eps, mf_bf16* x_mod, const KernelCtl& ctl,
                                  cudaStream_t st);
cudaError_t launch_rope(const mf_bf16* q, const mf_bf16* k, const int32_t* pos_ids, int32_t T,
                        int32_t H, int32_t D, const RopeTable& tab, mf_bf16* q_out,
                        mf_bf16* k_out, cudaStream_t st);
cudaError_t launch_gated_residual(const mf_bf16* x, const mf_bf16* o, const float* mod,
                                  const int32_t* tok_sample, const uint8_t* tok_mod, int32_t T,
                                  int32_t S, int32_t hid, mf_bf16* y, const KernelCtl& ctl,
                                  cudaStream_t st);

// Epilogue of the attention kernel.
struct AttnEpilogue {
  mf_bf16* o;             // [T][H][D] output (plain attention), or NULL
  float* lse;             // [H][T] or NULL
  const mf_bf16* x;       // gated residual: block input [T][H*D]
  const float* mod;       // [S][2][3][H*D]
  const uint8_t* tok_mod; // [T]
  mf_bf16* y;             // gated residual output [T][H*D], or NULL
};

// RoPE fused into the attention's load prologue: q is read unrotated and each
// Q tile is turned in shared memory before its first MMA (k arrives rotated by
// a RoPE pass over k alone), with (cos, sin) from a table of P positions x
// D / (2 axes) pair columns (one column set serves every axis: all axes use the
// same frequencies).
struct AttnRopeParams {
  const int32_t* pos_ids;  // [T][3]
  const void* tab;         // float2 [P][D / (2 axes)], from launch_rope_table
  int32_t P, axes;
};

// Writes the (cos, sin) table of P positions for head_dim D and rope_axes into
// tab (P * D / (2 rope_axes) float2) and fills r's tab, P and axes; the angles
// are computed as the standalone RoPE pass computes them.
cudaError_t launch_rope_table(int32_t D, int32_t rope_axes, float base, int32_t P, void* tab,
                              AttnRopeParams* r, cudaStream_t st);


// Work items of a pack, from host offsets: (sample, head, 256-row query block),
// or 512-row blocks for CTA pairs.
int32_t attention_work_items(const int32_t* cu_h, int32_t S, int32_t H, bool pair);

// rope == nullptr: q and k are already rotated. The gated epilogue (ep.y set)
// needs rope. pair: run head_dim 128 on CTA pairs (cta_group::2, M = 256).
cudaError_t launch_attention(const mf_bf16* q, const mf_bf16* k, const mf_bf16* v,
                             const int32_t* cu_seqlens_d, const int32_t* cu_seqlens_h, int32_t S,
                             int32_t T, int32_t H, int32_t D, float softmax_scale,
                             const AttnEpilogue& ep, const AttnRopeParams* rope, bool pair,
                             const KernelCtl& ctl, cudaStream_t st);

cudaError_t launch_selftest_exp2(const float* x, float* y, int32_t n, cudaStream_t st);
cudaError_t launch_selftest_wait(uint64_t limit_ns, const KernelCtl& ctl, cudaStream_t st);

}  // namespace mf
