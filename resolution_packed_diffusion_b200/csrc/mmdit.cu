// mmdit.cu -- one NR-MMDiT block forward around the packed joint-attention path,
// chained from the library's own kernels (host code only).
//
// Sources (page title, section): picx.dev "Mage-Flow" summary, Methodology >
// Native-Resolution MMDiT (modality-specific normalization, joint self-
// attention over the pack) and > Training Infrastructure (fused adaptive
// normalization / RoPE / gating). The pages do not give the block's wiring;
// the library takes the DiT-family block with two gated branches:
//   x1 = adaLN(x; mod_attn); q, k, v = x1 W{q,k,v}[m]^T
//   o = packed joint attention of RoPE(q), RoPE(k), v
//   y1 = x + gate_attn * (o Wo[m]^T)
//   x2 = adaLN(y1; mod_mlp); y = y1 + gate_mlp * (GELU(x2 Wup[m]^T) Wdown[m]^T)
// with m the token's modality. Every intermediate is stored in bf16 in the
// caller's workspace.
#include <cmath>
#include <cstdint>

#include "mf.h"

namespace {

inline size_t round_up256(size_t v) { return (v + 255) / 256 * 256; }

}  // namespace

extern "C" {

size_t mf_mmdit_workspace_size(int32_t T, int32_t H, int32_t D, int32_t F) {
  if (T < 0 || H < 1 || D < 1 || F < 1) return 0;
  const size_t row = static_cast<size_t>(T) * H * D * 2;
  return 9 * round_up256(row) + round_up256(static_cast<size_t>(T) * F * 2) +
         round_up256(mf_workspace_size(T, H, D, 1)) + 256;
}

mf_status mf_mmdit_block_fwd(const mf_bf16* x, const mf_bf16* Wq, const mf_bf16* Wk,
                             const mf_bf16* Wv, const mf_bf16* Wo, const mf_bf16* Wup,
                             const mf_bf16* Wdown, const float* mod_attn, const float* mod_mlp,
                             const mf_sample_desc* desc, const int32_t* cu_seqlens_d,
                             const int32_t* cu_seqlens_h, const int32_t* pos_ids,
                             const int32_t* tok_sample, const uint8_t* tok_mod, int32_t S,
                             int32_t H, int32_t D, int32_t F, int32_t rope_axes, float base,
                             float eps, mf_bf16* y, void* workspace, size_t ws_bytes,
                             cudaStream_t stream) {
  if (desc == nullptr || cu_seqlens_h == nullptr || S < 1 || S > MF_MAX_SAMPLES || H < 1 ||
      D < 1 || F < 256 || F % 256 != 0)
    return MF_ERR_INVALID;
  const int32_t hid = H * D;
  if (hid % 256 != 0) return MF_ERR_UNSUPPORTED;
  const int32_t T = cu_seqlens_h[S];
  if (T < 0 || T > MF_MAX_TOKENS) return MF_ERR_INVALID;
  if (T == 0) return MF_OK;
  if (workspace == nullptr || ws_bytes < mf_mmdit_workspace_size(T, H, D, F) ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
    return MF_ERR_INVALID;
  const size_t row = static_cast<size_t>(T) * hid * 2;
  auto overlaps = [](const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + nb && pb < pa + na;
  };
  if (y == nullptr || overlaps(y, row, x, row) || overlaps(y, row, workspace, ws_bytes))
    return MF_ERR_INVALID;
  uintptr_t p = (reinterpret_cast<uintptr_t>(workspace) + 255) / 256 * 256;
  auto take = [&](size_t bytes) {
    mf_bf16* b = reinterpret_cast<mf_bf16*>(p);
    p += round_up256(bytes);
    return b;
  };
  mf_bf16* x1 = take(row);
  mf_bf16* q = take(row);
  mf_bf16* k = take(row);
  mf_bf16* v = take(row);
  mf_bf16* o = take(row);
  mf_bf16* a = take(row);
  mf_bf16* y1 = take(row);
  mf_bf16* x2 = take(row);
  mf_bf16* mlp = take(row);
  mf_bf16* h = take(static_cast<size_t>(T) * F * 2);
  void* rope_ws = reinterpret_cast<void*>(p);
  const size_t rope_bytes = mf_workspace_size(T, H, D, 1);

  mf_status st;
#define MF_STEP(call)          \
  st = (call);                 \
  if (st != MF_OK) return st;
  // attention branch
  MF_STEP(mf_adaln_modulate(x, mod_attn, tok_sample, tok_mod, T, S, hid, eps, x1, stream));
  MF_STEP(mf_modality_linear(x1, Wq, tok_mod, desc, S, hid, hid, MF_ACT_NONE, q, stream));
  MF_STEP(mf_modality_linear(x1, Wk, tok_mod, desc, S, hid, hid, MF_ACT_NONE, k, stream));
  MF_STEP(mf_modality_linear(x1, Wv, tok_mod, desc, S, hid, hid, MF_ACT_NONE, v, stream));
  MF_STEP(mf_varlen_attn_fwd(q, k, v, cu_seqlens_d, cu_seqlens_h, S, H, D,
                             1.0f / std::sqrt(static_cast<float>(D)), pos_ids, rope_axes, base, o,
                             nullptr, rope_ws, rope_bytes, stream));
  MF_STEP(mf_modality_linear(o, Wo, tok_mod, desc, S, hid, hid, MF_ACT_NONE, a, stream));
  MF_STEP(mf_gated_residual(x, a, mod_attn, tok_sample, tok_mod, T, S, hid, y1, stream));
  // MLP branch
  MF_STEP(mf_adaln_modulate(y1, mod_mlp, tok_sample, tok_mod, T, S, hid, eps, x2, stream));
  MF_STEP(mf_modality_linear(x2, Wup, tok_mod, desc, S, hid, F, MF_ACT_GELU, h, stream));
  MF_STEP(mf_modality_linear(h, Wdown, tok_mod, desc, S, F, hid, MF_ACT_NONE, mlp, stream));
  MF_STEP(mf_gated_residual(y1, mlp, mod_mlp, tok_sample, tok_mod, T, S, hid, y, stream));
#undef MF_STEP
  return MF_OK;
}

}  // extern "C"
