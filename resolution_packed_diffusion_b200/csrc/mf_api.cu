// mf_api.cu -- the C ABI of libmf (declared in include/mf.h): argument checks,
// the per-device error word, workspace carving and kernel launches. No entry
// point allocates device memory; every buffer comes from the caller.
#include <cuda_runtime_api.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "mf.h"
#include "attn_bwd_internal.h"
#include "block_bwd_internal.h"
#include "cfg_internal.h"
#include "gemm_internal.h"
#include "mf_internal.h"
#include "vae_internal.h"

namespace mf {

// Per-device word where kernels record the first failure they detect.
__device__ int g_mf_error;

namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;

struct DeviceState {
  bool ready = false;
  int* err = nullptr;
  uint64_t wait_limit_ns = kDefaultWaitLimitNs;
  cudaEvent_t attn_start = nullptr;  // instrumentation (mf_set_attn_timing_events)
  cudaEvent_t attn_stop = nullptr;
  bool attn_pair = false;            // mf_set_attn_cta_pair
  bool linear_pair = true;           // mf_set_linear_cta_pair
  bool conv_pair = false;            // mf_set_conv_cta_pair
};

DeviceState g_state[kMaxDevices];
std::mutex g_mutex;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

thread_local char g_last_detail[256] = {0};

inline mf_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MF_OK;
  snprintf(g_last_detail, sizeof(g_last_detail), "%s: %s", cudaGetErrorName(e),
           cudaGetErrorString(e));
  return MF_ERR_CUDA;
}

bool valid_head_dim(int32_t D) { return D == 64 || D == 128; }

// Runs the attention launcher between the caller's timing events, if any.
// Runs the attention launcher (on CTA pairs when this device is set to) between
// the caller's timing events, if any.
cudaError_t timed_attention(const mf_bf16* q, const mf_bf16* k, const mf_bf16* v,
                            const int32_t* cu_d, const int32_t* cu_h, int32_t S, int32_t T,
                            int32_t H, int32_t D, float scale, const AttnEpilogue& ep,
                            const AttnRopeParams* rope, const KernelCtl& ctl, cudaStream_t st) {
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  bool pair = false;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices) {
    std::lock_guard<std::mutex> lock(g_mutex);
    e0 = g_state[dev].attn_start;
    e1 = g_state[dev].attn_stop;
    pair = g_state[dev].attn_pair;
  }
  if (e0 != nullptr) {
    cudaError_t e = cudaEventRecord(e0, st);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e =
      launch_attention(q, k, v, cu_d, cu_h, S, T, H, D, scale, ep, rope, pair, ctl, st);
  if (e != cudaSuccess) return e;
  if (e1 != nullptr) e = cudaEventRecord(e1, st);
  return e;
}

// Shared by mf_rope_apply and mf_rope_bwd: the backward turns by the negated
// angles (inverse frequencies negated in the table), which is the transpose
// of each pair rotation.
mf_status rope_call(const mf_bf16* q, const mf_bf16* k, const int32_t* pos_ids, int32_t T,
                    int32_t H, int32_t D, int32_t rope_axes, float base, mf_bf16* q_out,
                    mf_bf16* k_out, bool transpose, cudaStream_t stream) {
  if (T < 0 || T > MF_MAX_TOKENS || H < 1 || H > 128 || (rope_axes != 2 && rope_axes != 3) ||
      !(base > 0.f) || !std::isfinite(base))
    return MF_ERR_INVALID;
  if (!valid_head_dim(D)) return MF_ERR_UNSUPPORTED;
  if (q == nullptr && k == nullptr) return MF_ERR_INVALID;
  if ((q != nullptr) != (q_out != nullptr) || (k != nullptr) != (k_out != nullptr))
    return MF_ERR_INVALID;
  if (T == 0) return MF_OK;
  if (pos_ids == nullptr || !aligned16(q) || !aligned16(k) || !aligned16(q_out) ||
      !aligned16(k_out))
    return MF_ERR_INVALID;
  const size_t bytes = static_cast<size_t>(T) * H * D * 2;
  // in place is allowed; a partial overlap is not
  if (q && q != q_out && overlap(q, bytes, q_out, bytes)) return MF_ERR_INVALID;
  if (k && k != k_out && overlap(k, bytes, k_out, bytes)) return MF_ERR_INVALID;
  if (q_out && k_out && overlap(q_out, bytes, k_out, bytes)) return MF_ERR_INVALID;
  RopeTable tab;
  make_rope_table(D, rope_axes, base, &tab);
  if (transpose)
    for (float& f : tab.inv_freq) f = -f;
  return cuda_status(launch_rope(q, k, pos_ids, T, H, D, tab, q_out, k_out, stream));
}

// Carves the fused RoPE's workspace: the (cos, sin) table the attention turns
// Q tiles with, and the rotated k, written by the RoPE pass over k (the
// attention turns Q in its load prologue, K arrives rotated). Returns the k the
// attention reads.
cudaError_t prepare_fused_rope(const mf_bf16* k, const int32_t* pos_ids, int32_t T, int32_t H,
                               int32_t D, int32_t rope_axes, float base, void* workspace,
                               AttnRopeParams* rope, const mf_bf16** k_att, cudaStream_t st) {
  const uintptr_t w0 = round_up(reinterpret_cast<uintptr_t>(workspace), 256);
  rope->pos_ids = pos_ids;
  cudaError_t e = launch_rope_table(D, rope_axes, base, T, reinterpret_cast<void*>(w0), rope, st);
  if (e != cudaSuccess) return e;
  mf_bf16* kr = reinterpret_cast<mf_bf16*>(w0 + round_up(static_cast<size_t>(T) * (D / 4) * 8, 256));
  RopeTable tab;
  make_rope_table(D, rope_axes, base, &tab);
  *k_att = kr;
  return launch_rope(nullptr, k, pos_ids, T, H, D, tab, nullptr, kr, st);
}

}  // namespace

bool check_offsets(const int32_t* cu_h, int32_t S, int32_t* T) {
  if (cu_h == nullptr || cu_h[0] != 0) return false;
  for (int32_t s = 0; s < S; ++s)
    if (cu_h[s + 1] < cu_h[s]) return false;
  if (cu_h[S] > MF_MAX_TOKENS) return false;
  *T = cu_h[S];
  return true;
}

bool linear_cta_pair(bool* pair) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_mutex);
  *pair = g_state[dev].linear_pair;
  return true;
}

cudaError_t get_ctl(KernelCtl* ctl) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& d = g_state[dev];
  if (!d.ready) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_mf_error);
    if (e != cudaSuccess) return e;
    d.err = static_cast<int*>(p);
    d.ready = true;
  }
  ctl->err = d.err;
  ctl->wait_limit_ns = d.wait_limit_ns;
  return cudaSuccess;
}

}  // namespace mf

using namespace mf;

extern "C" {

int32_t mf_abi_version(void) { return MF_ABI_VERSION; }

const char* mf_last_error_detail(void) { return g_last_detail; }

const char* mf_status_string(mf_status s) {
  switch (s) {
    case MF_OK: return "MF_OK";
    case MF_ERR_INVALID: return "MF_ERR_INVALID";
    case MF_ERR_CUDA: return "MF_ERR_CUDA";
    case MF_ERR_TIMEOUT: return "MF_ERR_TIMEOUT";
    case MF_ERR_UNSUPPORTED: return "MF_ERR_UNSUPPORTED";
  }
  return "MF_ERR_UNKNOWN";
}

mf_status mf_pack_build(const mf_sample_desc* desc, int32_t S, int32_t rope_axes, int32_t budget,
                        int32_t* cu_seqlens_h, int32_t* cu_seqlens_d, int32_t* pos_ids_d,
                        int32_t* tok_sample_d, uint8_t* tok_mod_d, int32_t* T_out,
                        cudaStream_t stream) {
  if (S < 0 || S > MF_MAX_SAMPLES || (S > 0 && desc == nullptr) || cu_seqlens_h == nullptr ||
      T_out == nullptr || (rope_axes != 2 && rope_axes != 3) || budget < 0)
    return MF_ERR_INVALID;
  const int n_null = (cu_seqlens_d == nullptr) + (pos_ids_d == nullptr) +
                     (tok_sample_d == nullptr) + (tok_mod_d == nullptr);
  if (n_null != 0 && n_null != 4) return MF_ERR_INVALID;
  int64_t acc = 0;
  for (int32_t s = 0; s < S; ++s) {
    const mf_sample_desc& d = desc[s];
    if (d.frames < 0 || d.grid_h < 0 || d.grid_w < 0 || d.n_text < 0) return MF_ERR_INVALID;
    if (d.frames > (rope_axes == 2 ? 1 : 2)) return MF_ERR_INVALID;
    if (d.grid_h > MF_MAX_TOKENS || d.grid_w > MF_MAX_TOKENS || d.n_text > MF_MAX_TOKENS)
      return MF_ERR_INVALID;
    const int64_t n = static_cast<int64_t>(d.frames) * d.grid_h * d.grid_w + d.n_text;
    acc += n;
    if (acc > MF_MAX_TOKENS) return MF_ERR_INVALID;
  }
  if (budget > 0 && acc > budget) return MF_ERR_INVALID;
  PackParams p;
  p.S = S;
  p.T = static_cast<int32_t>(acc);
  p.cu[0] = 0;
  for (int32_t s = 0; s < S; ++s) {
    const mf_sample_desc& d = desc[s];
    p.cu[s + 1] = p.cu[s] + d.frames * d.grid_h * d.grid_w + d.n_text;
    p.frames[s] = d.frames;
    p.grid_h[s] = d.grid_h;
    p.grid_w[s] = d.grid_w;
  }
  for (int32_t s = 0; s <= S; ++s) cu_seqlens_h[s] = p.cu[s];
  *T_out = p.T;
  if (n_null == 4) return MF_OK;  // size query
  if (!aligned16(cu_seqlens_d) || !aligned16(pos_ids_d) || !aligned16(tok_sample_d) ||
      !aligned16(tok_mod_d))
    return MF_ERR_INVALID;
  return cuda_status(launch_pack_ids(p, cu_seqlens_d, pos_ids_d, tok_sample_d, tok_mod_d, stream));
}

mf_status mf_adaln_params(const float* c, const float* W, int32_t S, int32_t C, int32_t hid,
                          float* mod, cudaStream_t stream) {
  if (c == nullptr || W == nullptr || mod == nullptr || S < 1 || S > MF_MAX_SAMPLES || C < 1 ||
      C > 1024 || hid < 8 || hid % 8 != 0 || hid > 16384)
    return MF_ERR_INVALID;
  if (!aligned16(c) || !aligned16(W) || !aligned16(mod)) return MF_ERR_INVALID;
  return cuda_status(launch_adaln_params(c, W, S, C, hid, mod, stream));
}

mf_status mf_adaln_params_bwd(const float* dmod, const float* c, const float* W, int32_t S,
                              int32_t C, int32_t hid, float* dc, float* dW, cudaStream_t stream) {
  if (dmod == nullptr || c == nullptr || W == nullptr || (dc == nullptr && dW == nullptr) ||
      S < 1 || S > MF_MAX_SAMPLES || C < 1 || C > 1024 || hid < 8 || hid % 8 != 0 ||
      hid > 16384)
    return MF_ERR_INVALID;
  if (!aligned16(dmod) || !aligned16(c) || !aligned16(W) || !aligned16(dc) || !aligned16(dW))
    return MF_ERR_INVALID;
  const size_t mb = static_cast<size_t>(S) * 6 * hid * 4, cb = static_cast<size_t>(S) * C * 4,
               wb = static_cast<size_t>(C) * 6 * hid * 4;
  const void* ins[3] = {dmod, c, W};
  const size_t in_bytes[3] = {mb, cb, wb};
  for (int i = 0; i < 3; ++i) {
    if (dc && overlap(dc, cb, ins[i], in_bytes[i])) return MF_ERR_INVALID;
    if (dW && overlap(dW, wb, ins[i], in_bytes[i])) return MF_ERR_INVALID;
  }
  if (dc && dW && overlap(dc, cb, dW, wb)) return MF_ERR_INVALID;
  return cuda_status(launch_adaln_params_bwd(dmod, c, W, S, C, hid, dc, dW, stream));
}

mf_status mf_adaln_modulate(const mf_bf16* x, const float* mod, const int32_t* tok_sample,
                            const uint8_t* tok_mod, int32_t T, int32_t S, int32_t hid, float eps,
                            mf_bf16* x_mod, cudaStream_t stream) {
  if (T < 0 || T > MF_MAX_TOKENS || S < 1 || S > MF_MAX_SAMPLES || hid < 8 || hid % 8 != 0 ||
      !(eps >= 0.f) || !std::isfinite(eps))
    return MF_ERR_INVALID;
  if (hid > 4096) return MF_ERR_UNSUPPORTED;
  if (T == 0) return MF_OK;
  if (x == nullptr || mod == nullptr || tok_sample == nullptr || tok_mod == nullptr ||
      x_mod == nullptr || !aligned16(x) || !aligned16(mod) || !aligned16(x_mod))
    return MF_ERR_INVALID;
  const size_t bytes = static_cast<size_t>(T) * hid * 2;
  if (overlap(x, bytes, x_mod, bytes)) return MF_ERR_INVALID;
  KernelCtl ctl;
  if (cudaError_t ge = get_ctl(&ctl); ge != cudaSuccess) return cuda_status(ge);
  return cuda_status(
      launch_adaln_modulate(x, mod, tok_sample, tok_mod, T, S, hid, eps, x_mod, ctl, stream));
}


mf_status mf_rope_apply(const mf_bf16* q, const mf_bf16* k, const int32_t* pos_ids, int32_t T,
                        int32_t H, int32_t D, int32_t rope_axes, float base, mf_bf16* q_out,
                        mf_bf16* k_out, cudaStream_t stream) {
  return mf::rope_call(q, k, pos_ids, T, H, D, rope_axes, base, q_out, k_out, false, stream);
}

mf_status mf_rope_bwd(const mf_bf16* dq_r, const mf_bf16* dk_r, const int32_t* pos_ids,
                      int32_t T, int32_t H, int32_t D, int32_t rope_axes, float base,
                      mf_bf16* dq, mf_bf16* dk, cudaStream_t stream) {
  return mf::rope_call(dq_r, dk_r, pos_ids, T, H, D, rope_axes, base, dq, dk, true, stream);
}

// The workspace of the fused RoPE holds its (cos, sin) table, one row of
// D / (2 * rope_axes) <= D / 4 float2 per position, positions 0 .. T-1 (every
// position of a pack is below T: a sample's positions stay below its length),
// then the rotated k.
size_t mf_workspace_size(int32_t T, int32_t H, int32_t D, int32_t with_rope) {
  if (T <= 0 || H <= 0 || D <= 0 || !with_rope) return 0;
  return round_up(static_cast<size_t>(T) * (D / 4) * 8, 256) +
         round_up(static_cast<size_t>(T) * H * D * 2, 256) + 256;
}



mf_status mf_varlen_attn_fwd(const mf_bf16* q, const mf_bf16* k, const mf_bf16* v,
                             const int32_t* cu_seqlens_d, const int32_t* cu_seqlens_h, int32_t S,
                             int32_t H, int32_t D, float softmax_scale, const int32_t* pos_ids,
                             int32_t rope_axes, float base, mf_bf16* o, float* lse,
                             void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (S < 1 || S > MF_MAX_SAMPLES || H < 1 || H > 128 || !std::isfinite(softmax_scale) ||
      !(softmax_scale > 0.f))
    return MF_ERR_INVALID;
  if (!valid_head_dim(D)) return MF_ERR_UNSUPPORTED;
  int32_t T = 0;
  if (!check_offsets(cu_seqlens_h, S, &T)) return MF_ERR_INVALID;
  if (T == 0) return MF_OK;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || cu_seqlens_d == nullptr ||
      !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      !aligned16(cu_seqlens_d) || !aligned16(lse))
    return MF_ERR_INVALID;
  const size_t bytes = static_cast<size_t>(T) * H * D * 2;
  if (overlap(o, bytes, q, bytes) || overlap(o, bytes, k, bytes) || overlap(o, bytes, v, bytes))
    return MF_ERR_INVALID;
  if (lse && (overlap(lse, static_cast<size_t>(T) * H * 4, o, bytes)))
    return MF_ERR_INVALID;
  if (pos_ids != nullptr) {
    if ((rope_axes != 2 && rope_axes != 3) || !(base > 0.f) || !std::isfinite(base) ||
        !aligned16(pos_ids))
      return MF_ERR_INVALID;
    if (workspace == nullptr || !aligned16(workspace) || ws_bytes < mf_workspace_size(T, H, D, 1))
      return MF_ERR_INVALID;
    // the (cos, sin) table is written before the attention reads q, k, v and
    // pos_ids, and read while it writes o and lse
    const size_t ws = mf_workspace_size(T, H, D, 1);
    if (overlap(workspace, ws, q, bytes) || overlap(workspace, ws, k, bytes) ||
        overlap(workspace, ws, v, bytes) || overlap(workspace, ws, o, bytes) ||
        overlap(workspace, ws, pos_ids, static_cast<size_t>(T) * 12) ||
        (lse && overlap(workspace, ws, lse, static_cast<size_t>(T) * H * 4)))
      return MF_ERR_INVALID;
  }
  KernelCtl ctl;
  if (cudaError_t ge = get_ctl(&ctl); ge != cudaSuccess) return cuda_status(ge);
  AttnRopeParams rope{};
  const mf_bf16* ka = k;
  if (pos_ids != nullptr) {
    cudaError_t e = prepare_fused_rope(k, pos_ids, T, H, D, rope_axes, base, workspace, &rope,
                                       &ka, stream);
    if (e != cudaSuccess) return cuda_status(e);
  }
  AttnEpilogue ep{};
  ep.o = o;
  ep.lse = lse;
  return cuda_status(timed_attention(q, ka, v, cu_seqlens_d, cu_seqlens_h, S, T, H, D,
                                     softmax_scale, ep, pos_ids != nullptr ? &rope : nullptr,
                                     ctl, stream));
}

size_t mf_attn_bwd_workspace_size(int32_t T, int32_t S, int32_t H, int32_t D) {
  if (T < 0 || S < 1 || H < 1 || D < 1) return 0;
  return attn_bwd_workspace_bytes(T, S, H, D);
}

mf_status mf_varlen_attn_bwd(const mf_bf16* q, const mf_bf16* k, const mf_bf16* v,
                             const mf_bf16* o, const mf_bf16* d_o, const float* lse,
                             const int32_t* cu_seqlens_d, const int32_t* cu_seqlens_h, int32_t S,
                             int32_t H, int32_t D, float softmax_scale, mf_bf16* dq, mf_bf16* dk,
                             mf_bf16* dv, void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (S < 1 || S > MF_MAX_SAMPLES || H < 1 || H > 128 || !std::isfinite(softmax_scale) ||
      !(softmax_scale > 0.f))
    return MF_ERR_INVALID;
  if (!valid_head_dim(D)) return MF_ERR_UNSUPPORTED;
  int32_t T = 0;
  if (!check_offsets(cu_seqlens_h, S, &T)) return MF_ERR_INVALID;
  if (T == 0) return MF_OK;
  const mf_bf16* ins[5] = {q, k, v, o, d_o};
  mf_bf16* outs[3] = {dq, dk, dv};
  for (const mf_bf16* p : ins)
    if (p == nullptr || !aligned16(p)) return MF_ERR_INVALID;
  for (mf_bf16* p : outs)
    if (p == nullptr || !aligned16(p)) return MF_ERR_INVALID;
  if (lse == nullptr || !aligned16(lse) || cu_seqlens_d == nullptr) return MF_ERR_INVALID;
  if (workspace == nullptr || !aligned16(workspace) ||
      ws_bytes < mf_attn_bwd_workspace_size(T, S, H, D))
    return MF_ERR_INVALID;
  const size_t bytes = static_cast<size_t>(T) * H * D * 2;
  const size_t ws = mf_attn_bwd_workspace_size(T, S, H, D);
  for (int i = 0; i < 3; ++i) {
    for (const mf_bf16* p : ins)
      if (overlap(outs[i], bytes, p, bytes)) return MF_ERR_INVALID;
    for (int j = i + 1; j < 3; ++j)
      if (overlap(outs[i], bytes, outs[j], bytes)) return MF_ERR_INVALID;
    if (overlap(outs[i], bytes, workspace, ws) || overlap(outs[i], bytes, lse, static_cast<size_t>(T) * H * 4))
      return MF_ERR_INVALID;
  }
  for (const mf_bf16* p : ins)
    if (overlap(p, bytes, workspace, ws)) return MF_ERR_INVALID;
  if (overlap(lse, static_cast<size_t>(T) * H * 4, workspace, ws)) return MF_ERR_INVALID;
  KernelCtl ctl;
  if (cudaError_t ge = get_ctl(&ctl); ge != cudaSuccess) return cuda_status(ge);
  return cuda_status(launch_attention_bwd(q, k, v, o, d_o, lse, cu_seqlens_d, cu_seqlens_h, S, T,
                                          H, D, softmax_scale, dq, dk, dv, workspace, ctl,
                                          stream));
}

mf_status mf_gated_residual_bwd(const mf_bf16* dy, const mf_bf16* o, const float* mod,
                                const int32_t* tok_sample, const uint8_t* tok_mod, int32_t T,
                                int32_t S, int32_t hid, mf_bf16* d_o, float* dmod,
                                cudaStream_t stream) {
  if (T < 0 || T > MF_MAX_TOKENS || S < 1 || S > MF_MAX_SAMPLES || hid < 8 || hid % 8 != 0 ||
      hid > 65536)
    return MF_ERR_INVALID;
  if (mod == nullptr || dmod == nullptr || !aligned16(mod) || !aligned16(dmod))
    return MF_ERR_INVALID;
  const size_t mod_bytes = static_cast<size_t>(S) * 6 * hid * 4;
  if (overlap(mod, mod_bytes, dmod, mod_bytes)) return MF_ERR_INVALID;
  if (T > 0) {
    if (dy == nullptr || o == nullptr || d_o == nullptr || tok_sample == nullptr ||
        tok_mod == nullptr || !aligned16(dy) || !aligned16(o) || !aligned16(d_o))
      return MF_ERR_INVALID;
    const size_t bytes = static_cast<size_t>(T) * hid * 2;
    if (d_o != dy && overlap(d_o, bytes, dy, bytes)) return MF_ERR_INVALID;
    if (overlap(d_o, bytes, o, bytes) || overlap(d_o, bytes, dmod, mod_bytes) ||
        overlap(d_o, bytes, mod, mod_bytes))
      return MF_ERR_INVALID;
    // dmod is zeroed before dy and o are read: it must not overlap them
    if (overlap(dmod, mod_bytes, dy, bytes) || overlap(dmod, mod_bytes, o, bytes))
      return MF_ERR_INVALID;
  }
  KernelCtl ctl;
  if (cudaError_t ge = get_ctl(&ctl); ge != cudaSuccess) return cuda_status(ge);
  return cuda_status(launch_gated_residual_bwd(dy, o, mod, tok_sample, tok_mod, T, S, hid, d_o,
                                               dmod, ctl, stream));
}

size_t mf_adaln_bwd_workspace_size(int32_t T) {
  if (T <= 0) return 0;
  return round_up(static_cast<size_t>(T) * 8, 256) + 256;
}

mf_status mf_adaln_modulate_bwd(const mf_bf16* dx_mod, const mf_bf16* x, const float* mod,
                                const int32_t* tok_sample, const uint8_t* tok_mod,
                                const mf_bf16* resid, int32_t T, int32_t S, int32_t hid,
                                float eps, mf_bf16* dx, float* dmod, void* workspace,
                                size_t ws_bytes, cudaStream_t stream) {
  if (T < 0 || T > MF_MAX_TOKENS || S < 1 || S > MF_MAX_SAMPLES || hid < 8 || hid % 8 != 0 ||
      hid > 65536 || !(eps > 0.f) || !std::isfinite(eps))
    return MF_ERR_INVALID;
  if (mod == nullptr || dmod == nullptr || !aligned16(mod) || !aligned16(dmod))
    return MF_ERR_INVALID;
  const size_t mod_bytes = static_cast<size_t>(S) * 6 * hid * 4;
  if (overlap(mod, mod_bytes, dmod, mod_bytes)) return MF_ERR_INVALID;
  float* stats = nullptr;
  if (T > 0) {
    if (dx_mod == nullptr || x == nullptr || dx == nullptr || tok_sample == nullptr ||
        tok_mod == nullptr || !aligned16(dx_mod) || !aligned16(x) || !aligned16(dx) ||
        (resid != nullptr && !aligned16(resid)))
      return MF_ERR_INVALID;
    if (workspace == nullptr || !aligned16(workspace) || ws_bytes < mf_adaln_bwd_workspace_size(T))
      return MF_ERR_INVALID;
    const size_t bytes = static_cast<size_t>(T) * hid * 2;
    const size_t ws = mf_adaln_bwd_workspace_size(T);
    // dx may equal resid (in place); it must not touch x, dx_mod, dmod or the workspace
    if (resid != nullptr && dx != resid && overlap(dx, bytes, resid, bytes)) return MF_ERR_INVALID;
    if (overlap(dx, bytes, x, bytes) || overlap(dx, bytes, dx_mod, bytes) ||
        overlap(dx, bytes, dmod, mod_bytes) || overlap(dx, bytes, workspace, ws) ||
        overlap(dx, bytes, mod, mod_bytes) || overlap(dmod, mod_bytes, workspace, ws))
      return MF_ERR_INVALID;
    // dmod is zeroed and the row statistics written before the inputs are read
    if (overlap(dmod, mod_bytes, x, bytes) || overlap(dmod, mod_bytes, dx_mod, bytes) ||
        (resid != nullptr && overlap(dmod, mod_bytes, resid, bytes)) ||
        overlap(workspace, ws, x, bytes) || overlap(workspace, ws, dx_mod, bytes) ||
        overlap(workspace, ws, mod, mod_bytes) ||
        (resid != nullptr && overlap(workspace, ws, resid, bytes)))
      return MF_ERR_INVALID;
    stats = reinterpret_cast<float*>(round_up(reinterpret_cast<uintptr_t>(workspace), 256));
  }
  KernelCtl ctl;
  if (cudaError_t ge = get_ctl(&ctl); ge != cudaSuccess) return cuda_status(ge);
  return cuda_status(launch_adaln_modulate_bwd(dx_mod, x, mod, tok_sample, tok_mod, resid, T, S,
                                               hid, eps, dx, dmod, stats, ctl, stream));
}

mf_status mf_gated_residual(const mf_bf16* x, const mf_bf16* o, const float* mod,
                            const int32_t* tok_sample, const uint8_t* tok_mod, int32_t T,
                            int32_t S, int32_t hid, mf_bf16* y, cudaStream_t stream) {
  if (T < 0 || T > MF_MAX_TOKENS || S < 1 || S > MF_MAX_SAMPLES || hid < 8 || hid % 8 != 0)
    return MF_ERR_INVALID;
  if (T == 0) return MF_OK;
  if (x == nullptr || o == nullptr || mod == nullptr || tok_sample == nullptr ||
      tok_mod == nullptr || y == nullptr || !aligned16(x) || !aligned16(o) || !aligned16(mod) ||
      !aligned16(y))
    return MF_ERR_INVALID;
  const size_t bytes = static_cast<size_t>(T) * hid * 2;
  if (y != x && overlap(x, bytes, y, bytes)) return MF_ERR_INVALID;
  if (overlap(o, bytes, y, bytes)) return MF_ERR_INVALID;
  KernelCtl ctl;
  if (cudaError_t ge = get_ctl(&ctl); ge != cudaSuccess) return cuda_status(ge);
  return cuda_status(
      launch_gated_residual(x, o, mod, tok_sample, tok_mod, T, S, hid, y, ctl, stream));
}

mf_status mf_block_fwd(const mf_bf16* x, const mf_bf16* q, const mf_bf16* k, const mf_bf16* v,
                       const float* mod, const int32_t* cu_seqlens_d, const int32_t* cu_seqlens_h,
                       const int32_t* pos_ids, const int32_t* tok_sample, const uint8_t* tok_mod,
                       int32_t S, int32_t H, int32_t D, int32_t rope_axes, float base, float eps,
                       mf_bf16* x_mod, mf_bf16* y, void* workspace, size_t ws_bytes,
                       cudaStream_t stream) {
  if (S < 1 || S > MF_MAX_SAMPLES || H < 1 || H > 128 || (rope_axes != 2 && rope_axes != 3) ||
      !(base > 0.f) || !std::isfinite(base) || !(eps >= 0.f) || !std::isfinite(eps))
    return MF_ERR_INVALID;
  if (!valid_head_dim(D) || H * D > 4096) return MF_ERR_UNSUPPORTED;
  int32_t T = 0;
  if (!check_offsets(cu_seqlens_h, S, &T)) return MF_ERR_INVALID;
  if (T == 0) return MF_OK;
  const int32_t hid = H * D;
  if (x == nullptr || q == nullptr || k == nullptr || v == nullptr || mod == nullptr ||
      cu_seqlens_d == nullptr || pos_ids == nullptr || tok_sample == nullptr ||
      tok_mod == nullptr || x_mod == nullptr || y == nullptr || workspace == nullptr)
    return MF_ERR_INVALID;
  if (!aligned16(x) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(mod) ||
      !aligned16(cu_seqlens_d) || !aligned16(x_mod) || !aligned16(y) || !aligned16(workspace) ||
      !aligned16(pos_ids))
    return MF_ERR_INVALID;
  if (ws_bytes < mf_workspace_size(T, H, D, 1)) return MF_ERR_INVALID;
  const size_t bytes = static_cast<size_t>(T) * hid * 2;
  const void* ins[4] = {x, q, k, v};
  for (const void* in : ins)
    if (overlap(in, bytes, x_mod, bytes) || overlap(in, bytes, y, bytes)) return MF_ERR_INVALID;
  if (overlap(x_mod, bytes, y, bytes)) return MF_ERR_INVALID;
  // The (cos, sin) table is written into the workspace before the attention
  // reads q, k, v and pos_ids, and the fused epilogue reads x and mod while y
  // is written: the workspace and the outputs must stay clear of every input.
  const size_t ws = mf_workspace_size(T, H, D, 1);
  const size_t mod_bytes = static_cast<size_t>(S) * 6 * hid * 4;
  for (const void* in : ins)
    if (overlap(workspace, ws, in, bytes)) return MF_ERR_INVALID;
  if (overlap(workspace, ws, mod, mod_bytes) || overlap(workspace, ws, x_mod, bytes) ||
      overlap(workspace, ws, y, bytes) || overlap(workspace, ws, pos_ids, static_cast<size_t>(T) * 12))
    return MF_ERR_INVALID;
  if (overlap(x_mod, bytes, mod, mod_bytes) || overlap(y, bytes, mod, mod_bytes))
    return MF_ERR_INVALID;
  KernelCtl ctl;
  if (cudaError_t ge = get_ctl(&ctl); ge != cudaSuccess) return cuda_status(ge);
  cudaError_t e =
      launch_adaln_modulate(x, mod, tok_sample, tok_mod, T, S, hid, eps, x_mod, ctl, stream);
  if (e != cudaSuccess) return cuda_status(e);
  // RoPE in the attention's load prologue: Q and K tiles are turned in shared
  // memory with (cos, sin) from a per-position table in the workspace
  AttnRopeParams rope{};
  const mf_bf16* ka = k;
  e = prepare_fused_rope(k, pos_ids, T, H, D, rope_axes, base, workspace, &rope, &ka, stream);
  if (e != cudaSuccess) return cuda_status(e);
  AttnEpilogue ep{};
  ep.x = x;
  ep.mod = mod;
  ep.tok_mod = tok_mod;
  ep.y = y;
  return cuda_status(timed_attention(q, ka, v, cu_seqlens_d, cu_seqlens_h, S, T, H, D,
                                     1.0f / std::sqrt(static_cast<float>(D)), ep, &rope,
                                     ctl, stream));
}

mf_status mf_cfg_combine(const mf_bf16* v, const mf_sample_desc* desc, int32_t S,
                         const mf_cfg_pair* pairs, int32_t P, int32_t C, float w, mf_bf16* out,
                         cudaStream_t stream) {
  if (desc == nullptr || pairs == nullptr || S < 1 || S > MF_MAX_SAMPLES || P < 1 ||
      P > kMaxCfgPairs || C < 8 || C % 8 != 0 || !std::isfinite(w))
    return MF_ERR_INVALID;
  // offsets and image-token counts of the samples, from the descriptors
  static thread_local CfgTable tab;
  int64_t cu[MF_MAX_SAMPLES + 1];
  int64_t n_img[MF_MAX_SAMPLES];
  cu[0] = 0;
  for (int32_t s = 0; s < S; ++s) {
    const mf_sample_desc& d = desc[s];
    if (d.frames < 0 || d.grid_h < 0 || d.grid_w < 0 || d.n_text < 0) return MF_ERR_INVALID;
    n_img[s] = static_cast<int64_t>(d.frames) * d.grid_h * d.grid_w;
    cu[s + 1] = cu[s] + n_img[s] + d.n_text;
    if (cu[s + 1] > MF_MAX_TOKENS) return MF_ERR_INVALID;
  }
  const int64_t T = cu[S];
  int64_t rows = 0;
  tab.P = P;
  for (int32_t p = 0; p < P; ++p) {
    const int32_t c = pairs[p].cond, u = pairs[p].uncond;
    if (c < 0 || c >= S || u < 0 || u >= S || c == u || n_img[c] != n_img[u])
      return MF_ERR_INVALID;
    tab.out0[p] = static_cast<int32_t>(rows);
    tab.cond0[p] = static_cast<int32_t>(cu[c]);
    tab.uncond0[p] = static_cast<int32_t>(cu[u]);
    rows += n_img[c];
    if (rows > MF_MAX_TOKENS) return MF_ERR_INVALID;
  }
  tab.out0[P] = static_cast<int32_t>(rows);
  if (rows == 0) return MF_OK;
  if (v == nullptr || out == nullptr || !aligned16(v) || !aligned16(out)) return MF_ERR_INVALID;
  if (overlap(v, static_cast<size_t>(T) * C * 2, out, static_cast<size_t>(rows) * C * 2))
    return MF_ERR_INVALID;
  return cuda_status(launch_cfg_combine(v, tab, C, w, out, stream));
}

mf_status mf_modality_linear(const mf_bf16* x, const mf_bf16* W, const uint8_t* tok_mod,
                             const mf_sample_desc* desc, int32_t S, int32_t K, int32_t N,
                             int32_t act, mf_bf16* out, cudaStream_t stream) {
  if (desc == nullptr || S < 1 || S > MF_MAX_SAMPLES || K < 64 || K % 64 != 0 || N < 256 ||
      N % 256 != 0 || N > (1 << 20) || (act != MF_ACT_NONE && act != MF_ACT_GELU))
    return MF_ERR_INVALID;
  int32_t n_img[MF_MAX_SAMPLES], n_txt[MF_MAX_SAMPLES];
  int64_t T = 0;
  for (int32_t s = 0; s < S; ++s) {
    const mf_sample_desc& d = desc[s];
    if (d.frames < 0 || d.grid_h < 0 || d.grid_w < 0 || d.n_text < 0) return MF_ERR_INVALID;
    const int64_t ni = static_cast<int64_t>(d.frames) * d.grid_h * d.grid_w;
    if (ni > MF_MAX_TOKENS) return MF_ERR_INVALID;
    n_img[s] = static_cast<int32_t>(ni);
    n_txt[s] = d.n_text;
    T += ni + d.n_text;
    if (T > MF_MAX_TOKENS) return MF_ERR_INVALID;
  }
  if (T == 0) return MF_OK;
  if (x == nullptr || W == nullptr || tok_mod == nullptr || out == nullptr || !aligned16(x) ||
      !aligned16(W) || !aligned16(out))
    return MF_ERR_INVALID;
  const size_t xb = static_cast<size_t>(T) * K * 2, wb = static_cast<size_t>(2) * N * K * 2,
               ob = static_cast<size_t>(T) * N * 2;
  if (overlap(out, ob, x, xb) || overlap(out, ob, W, wb)) return MF_ERR_INVALID;
  KernelCtl ctl;
  if (cudaError_t ge = get_ctl(&ctl); ge != cudaSuccess) return cuda_status(ge);
  bool pair = false;
  if (!linear_cta_pair(&pair)) return MF_ERR_CUDA;
  static thread_local GemmJobs jobs;
  if (!build_gemm_jobs(n_img, n_txt, S, static_cast<int32_t>(T), gemm_job_rows(pair), &jobs))
    return MF_ERR_UNSUPPORTED;
  return cuda_status(launch_modality_linear(x, W, tok_mod, jobs, pair, static_cast<int32_t>(T), K,
                                            N, act, out, ctl, stream));
}

namespace {
// Channel counts the VAE kernels take: a multiple of 64 (one 128-byte K atom of
// the conv) whose 8-channel vector count divides 256 (the statistics pass).
bool vae_channels_ok(int32_t C) {
  return C >= 64 && C <= 2048 && (C & (C - 1)) == 0;
}
bool vae_shape_ok(int32_t N, int32_t H, int32_t W) {
  return N >= 1 && H >= 1 && W >= 1 && static_cast<int64_t>(N) * H * W < (int64_t{1} << 31) &&
         H <= (1 << 20) && W <= (1 << 20);
}

// The conv kernel form chosen for the current device (mf_set_conv_cta_pair).
bool conv_pair_setting(bool* pair) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_mutex);
  *pair = g_state[dev].conv_pair;
  return true;
}
}  // namespace

size_t mf_gn_workspace_size(int32_t N, int32_t H, int32_t W, int32_t G) {
  if (!vae_shape_ok(N, H, W) || G < 1) return 0;
  return gn_workspace_bytes(N, H, W, G) + 256;
}

mf_status mf_group_norm_silu(const mf_bf16* x, const float* gamma, const float* beta, int32_t N,
                             int32_t H, int32_t W, int32_t C, int32_t G, float eps, mf_bf16* y,
                             void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (x == nullptr || gamma == nullptr || beta == nullptr || y == nullptr ||
      workspace == nullptr || G < 1 || !(eps >= 0.f) || !std::isfinite(eps))
    return MF_ERR_INVALID;
  if (!vae_shape_ok(N, H, W)) return MF_ERR_INVALID;
  if (!vae_channels_ok(C) || C % G != 0 || (C / G) % 8 != 0) return MF_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(beta) || !aligned16(y) ||
      !aligned16(workspace))
    return MF_ERR_INVALID;
  const size_t ws = mf_gn_workspace_size(N, H, W, G);
  if (ws_bytes < ws) return MF_ERR_INVALID;
  const size_t bytes = static_cast<size_t>(N) * H * W * C * 2;
  if (overlap(x, bytes, y, bytes) || overlap(workspace, ws, x, bytes) ||
      overlap(workspace, ws, y, bytes) || overlap(y, bytes, gamma, C * 4) ||
      overlap(y, bytes, beta, C * 4))
    return MF_ERR_INVALID;
  void* w0 = reinterpret_cast<void*>(round_up(reinterpret_cast<uintptr_t>(workspace), 256));
  return cuda_status(launch_group_norm_silu(x, gamma, beta, N, H, W, C, G, eps, y, w0, stream));
}

mf_status mf_conv3x3(const mf_bf16* x, const mf_bf16* Wt, const float* bias,
                     const mf_bf16* residual, int32_t N, int32_t H, int32_t W, int32_t Cin,
                     int32_t Cout, mf_bf16* y, cudaStream_t stream) {
  if (x == nullptr || Wt == nullptr || y == nullptr) return MF_ERR_INVALID;
  if (!vae_shape_ok(N, H, W)) return MF_ERR_INVALID;
  if (!vae_channels_ok(Cin) || !vae_channels_ok(Cout)) return MF_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(Wt) || !aligned16(y) || !aligned16(bias) ||
      !aligned16(residual))
    return MF_ERR_INVALID;
  const size_t xb = static_cast<size_t>(N) * H * W * Cin * 2;
  const size_t yb = static_cast<size_t>(N) * H * W * Cout * 2;
  const size_t wb = static_cast<size_t>(Cout) * 9 * Cin * 2;
  if (overlap(y, yb, x, xb) || overlap(y, yb, Wt, wb) || (bias && overlap(y, yb, bias, Cout * 4)))
    return MF_ERR_INVALID;
  if (residual != nullptr && residual != y && overlap(residual, yb, y, yb)) return MF_ERR_INVALID;
  KernelCtl ctl;
  if (cudaError_t ge = get_ctl(&ctl); ge != cudaSuccess) return cuda_status(ge);
  bool pair = false;
  if (!conv_pair_setting(&pair)) return MF_ERR_CUDA;
  return cuda_status(
      launch_conv3x3(x, Wt, bias, residual, N, H, W, Cin, Cout, y, pair, ctl, stream));
}

size_t mf_vae_block_workspace_size(int32_t N, int32_t H, int32_t W, int32_t C, int32_t G) {
  if (!vae_shape_ok(N, H, W) || C < 1 || G < 1) return 0;
  const size_t act = round_up(static_cast<size_t>(N) * H * W * C * 2, 256);
  return 2 * act + mf_gn_workspace_size(N, H, W, G) + 256;
}

mf_status mf_vae_res_block(const mf_bf16* x, const float* gamma1, const float* beta1,
                           const mf_bf16* W1, const float* c1, const float* gamma2,
                           const float* beta2, const mf_bf16* W2, const float* c2, int32_t N,
                           int32_t H, int32_t W, int32_t C, int32_t G, float eps, mf_bf16* y,
                           void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (x == nullptr || gamma1 == nullptr || beta1 == nullptr || W1 == nullptr ||
      gamma2 == nullptr || beta2 == nullptr || W2 == nullptr || y == nullptr ||
      workspace == nullptr || G < 1 || !(eps >= 0.f) || !std::isfinite(eps))
    return MF_ERR_INVALID;
  if (!vae_shape_ok(N, H, W)) return MF_ERR_INVALID;
  if (!vae_channels_ok(C) || C % G != 0 || (C / G) % 8 != 0) return MF_ERR_UNSUPPORTED;
  const void* ptrs[10] = {x, gamma1, beta1, W1, c1, gamma2, beta2, W2, c2, y};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MF_ERR_INVALID;
  if (!aligned16(workspace)) return MF_ERR_INVALID;
  const size_t ws = mf_vae_block_workspace_size(N, H, W, C, G);
  if (ws_bytes < ws) return MF_ERR_INVALID;
  const size_t ab = static_cast<size_t>(N) * H * W * C * 2;
  const size_t wb = static_cast<size_t>(C) * 9 * C * 2;
  if (overlap(y, ab, x, ab) || overlap(y, ab, W1, wb) || overlap(y, ab, W2, wb) ||
      overlap(y, ab, workspace, ws) || overlap(workspace, ws, x, ab) ||
      overlap(workspace, ws, W1, wb) || overlap(workspace, ws, W2, wb))
    return MF_ERR_INVALID;
  KernelCtl ctl;
  if (cudaError_t ge = get_ctl(&ctl); ge != cudaSuccess) return cuda_status(ge);
  bool pair = false;
  if (!conv_pair_setting(&pair)) return MF_ERR_CUDA;
  const uintptr_t w0 = round_up(reinterpret_cast<uintptr_t>(workspace), 256);
  mf_bf16* a = reinterpret_cast<mf_bf16*>(w0);                       // SiLU(GN(.)), reused
  mf_bf16* h = reinterpret_cast<mf_bf16*>(w0 + round_up(ab, 256));   // first conv's output
  void* gws = reinterpret_cast<void*>(w0 + 2 * round_up(ab, 256));   // GroupNorm statistics
  cudaError_t e = launch_group_norm_silu(x, gamma1, beta1, N, H, W, C, G, eps, a, gws, stream);
  if (e != cudaSuccess) return cuda_status(e);
  e = launch_conv3x3(a, W1, c1, nullptr, N, H, W, C, C, h, pair, ctl, stream);
  if (e != cudaSuccess) return cuda_status(e);
  e = launch_group_norm_silu(h, gamma2, beta2, N, H, W, C, G, eps, a, gws, stream);
  if (e != cudaSuccess) return cuda_status(e);
  return cuda_status(launch_conv3x3(a, W2, c2, x, N, H, W, C, C, y, pair, ctl, stream));
}

mf_status mf_get_error(cudaStream_t stream) {
  cudaError_t se = cudaStreamSynchronize(stream);
  if (se != cudaSuccess) return cuda_status(se);
  KernelCtl ctl;
  if (cudaError_t ge = get_ctl(&ctl); ge != cudaSuccess) return cuda_status(ge);
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_mf_error, sizeof(int)) != cudaSuccess) return MF_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_mf_error, &zero, sizeof(int)) != cudaSuccess) return MF_ERR_CUDA;
  return static_cast<mf_status>(v);
}

mf_status mf_set_wait_limit_ns(uint64_t ns) {
  if (ns == 0) return MF_ERR_INVALID;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MF_ERR_CUDA;
  if (dev < 0 || dev >= 64) return MF_ERR_INVALID;
  std::lock_guard<std::mutex> lock(g_mutex);
  g_state[dev].wait_limit_ns = ns;
  return MF_OK;
}

mf_status mf_set_attn_cta_pair(int32_t enable) {
  if (enable != 0 && enable != 1) return MF_ERR_INVALID;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MF_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MF_ERR_INVALID;
  std::lock_guard<std::mutex> lock(g_mutex);
  g_state[dev].attn_pair = enable != 0;
  return MF_OK;
}

mf_status mf_set_linear_cta_pair(int32_t enable) {
  if (enable != 0 && enable != 1) return MF_ERR_INVALID;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MF_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MF_ERR_INVALID;
  std::lock_guard<std::mutex> lock(g_mutex);
  g_state[dev].linear_pair = enable != 0;
  return MF_OK;
}

mf_status mf_set_conv_cta_pair(int32_t enable) {
  if (enable != 0 && enable != 1) return MF_ERR_INVALID;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MF_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MF_ERR_INVALID;
  std::lock_guard<std::mutex> lock(g_mutex);
  g_state[dev].conv_pair = enable != 0;
  return MF_OK;
}

mf_status mf_set_attn_timing_events(cudaEvent_t start, cudaEvent_t stop) {
  if ((start == nullptr) != (stop == nullptr)) return MF_ERR_INVALID;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MF_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MF_ERR_INVALID;
  std::lock_guard<std::mutex> lock(g_mutex);
  g_state[dev].attn_start = start;
  g_state[dev].attn_stop = stop;
  return MF_OK;
}

mf_status mf_selftest_exp2_poly(const float* x, float* y, int32_t n, cudaStream_t stream) {
  if (n < 0 || (n > 0 && (x == nullptr || y == nullptr))) return MF_ERR_INVALID;
  return cuda_status(launch_selftest_exp2(x, y, n, stream));
}

mf_status mf_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return MF_ERR_INVALID;
  KernelCtl ctl;
  if (cudaError_t ge = get_ctl(&ctl); ge != cudaSuccess) return cuda_status(ge);
  return cuda_status(launch_selftest_wait(limit_ns, ctl, stream));
}

}  // extern "C"
