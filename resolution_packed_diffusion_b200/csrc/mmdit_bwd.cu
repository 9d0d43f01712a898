// mmdit_bwd.cu -- backward of one NR-MMDiT block (the forward is mmdit.cu): the
// forward's intermediates recomputed in the caller's workspace, then the chain
// rule through both gated branches, with every product on the library's
// tcgen05 linear kernel.
//
// Sources (page title, section): picx.dev "Mage-Flow" summary, Methodology >
// Native-Resolution MMDiT (modality-specific projections, joint attention) and
// > Training Infrastructure (the packed model is trained; its step-time and MFU
// figures are training steps). The block is the one mmdit.cu computes:
//   x1 = adaLN(x; mod_attn); q, k, v = x1 W{q,k,v}[m]^T
//   o = packed joint attention of RoPE(q), RoPE(k), v
//   y1 = x + gate_attn * (o Wo[m]^T)
//   x2 = adaLN(y1; mod_mlp); z = x2 Wup[m]^T; y = y1 + gate_mlp * (GELU(z) Wdown[m]^T)
// A linear layer out[t] = in[t] W[m]^T has the gradients
//   d_in[t] = d_out[t] W[m]            (the linear kernel on W[m]^T, stored once)
//   dW[m]   = sum over modality-m tokens of d_out[t]^T in[t]
// the second as the linear kernel on two transposes that gather the
// modality's token columns: rows d_out^T [N][T_m], inner dimension T_m
// (zero-padded to a multiple of 64), weights in^T [K][T_m].
//
// Kernels here: transpose_kernel (bf16 tiles of 64 x 64 through shared memory,
// source rows picked by runs of consecutive tokens), gelu_kernel /
// gelu_bwd_kernel (the tanh-form GELU and its derivative, 16-byte vectors),
// pack3_kernel (dq | dk | dv side by side, so that one product over an inner
// dimension of 3 hid forms dx1 = dq Wq + dk Wk + dv Wv with one fp32 sum), and
// zero_kernel.
#include <cmath>
#include <cstdint>

#include <cuda_bf16.h>

#include "gemm_internal.h"
#include "mf.h"
#include "mf_internal.h"
#include "mf_ptx.cuh"

namespace mf {
namespace {

constexpr int kTile = 64;

// Runs of consecutive source rows: destination column j in [dst0[r], dst0[r+1])
// reads source row src0[r] + (j - dst0[r]); columns from dst0[n] on are zero.
struct RunTable {
  int32_t n;
  int32_t src0[MF_MAX_SAMPLES];
  int32_t dst0[MF_MAX_SAMPLES + 1];
};

__device__ __forceinline__ int src_row(const RunTable& rt, int j) {
  if (j >= rt.dst0[rt.n]) return -1;
  int lo = 0, hi = rt.n - 1;  // last run with dst0[r] <= j
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (rt.dst0[mid] <= j) lo = mid; else hi = mid - 1;
  }
  return rt.src0[lo] + (j - rt.dst0[lo]);
}

// dst[c][dst_col0 + j] = src[row(j)][c] for c < C, j < n_pad (zero where row(j)
// is -1). One CTA per 64 x 64 tile: grid (n_pad / 64, C / 64).
__global__ void __launch_bounds__(256) transpose_kernel(const uint16_t* __restrict__ src,
                                                        int64_t src_ld, const RunTable rt,
                                                        uint16_t* __restrict__ dst, int64_t dst_ld,
                                                        int32_t dst_col0) {
  __shared__ uint16_t tile[kTile][kTile + 2];
  const int j0 = blockIdx.x * kTile, c0 = blockIdx.y * kTile;
  // load: 64 source rows x 64 columns, one 16-byte vector per thread and pass
  for (int v = threadIdx.x; v < kTile * kTile / 8; v += blockDim.x) {
    const int jr = v >> 3, c8 = (v & 7) * 8;
    const int r = src_row(rt, j0 + jr);
    uint4 u = make_uint4(0, 0, 0, 0);
    if (r >= 0) u = __ldg(reinterpret_cast<const uint4*>(src + r * src_ld + c0 + c8));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      tile[jr][c8 + 2 * e] = static_cast<uint16_t>(w[e] & 0xFFFFu);
      tile[jr][c8 + 2 * e + 1] = static_cast<uint16_t>(w[e] >> 16);
    }
  }
  __syncthreads();
  // store: 64 destination rows (source columns) x 64 columns
  for (int v = threadIdx.x; v < kTile * kTile / 8; v += blockDim.x) {
    const int cr = v >> 3, j8 = (v & 7) * 8;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      w[e] = static_cast<uint32_t>(tile[j8 + 2 * e][cr]) |
             (static_cast<uint32_t>(tile[j8 + 2 * e + 1][cr]) << 16);
    *reinterpret_cast<uint4*>(dst + (c0 + cr) * dst_ld + dst_col0 + j0 + j8) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

constexpr float kSqrt2OverPi = 0.7978845608028654f;
constexpr float kGeluCubic = 0.044715f;

// h = GELU(z), tanh form: 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))).
__global__ void __launch_bounds__(256) gelu_kernel(const uint4* __restrict__ z, int64_t n8,
                                                   uint4* __restrict__ h) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float f[8];
    unpack8(__ldg(z + i), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float u = kSqrt2OverPi * fmaf(kGeluCubic * f[e], f[e] * f[e], f[e]);
      f[e] = 0.5f * f[e] * (1.f + tanhf(u));
    }
    h[i] = pack8(f);
  }
}

// dz = dh * GELU'(z), GELU'(z) = 0.5 (1 + th) + 0.5 z (1 - th^2) sqrt(2/pi)
// (1 + 3 * 0.044715 z^2), th = tanh(sqrt(2/pi) (z + 0.044715 z^3)). dz may equal dh.
__global__ void __launch_bounds__(256) gelu_bwd_kernel(const uint4* __restrict__ z,
                                                       const uint4* dh, int64_t n8, uint4* dz) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float fz[8], fg[8];
    unpack8(__ldg(z + i), fz);
    unpack8(dh[i], fg);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x = fz[e];
      const float th = tanhf(kSqrt2OverPi * fmaf(kGeluCubic * x, x * x, x));
      const float d = 0.5f * (1.f + th) +
                      0.5f * x * (1.f - th * th) * kSqrt2OverPi * fmaf(3.f * kGeluCubic, x * x, 1.f);
      fg[e] *= d;
    }
    dz[i] = pack8(fg);
  }
}

// out[t][j * hid + c] = in_j[t][c] for j = 0, 1, 2.
__global__ void __launch_bounds__(256) pack3_kernel(const uint4* __restrict__ a,
                                                    const uint4* __restrict__ b,
                                                    const uint4* __restrict__ c, int64_t T,
                                                    int32_t hid8, uint4* __restrict__ out) {
  const int64_t n = T * hid8;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / hid8;
    const int64_t col = i - t * hid8;
    uint4* row = out + t * 3 * hid8 + col;
    row[0] = __ldg(a + i);
    row[hid8] = __ldg(b + i);
    row[2 * hid8] = __ldg(c + i);
  }
}

__global__ void __launch_bounds__(256) zero_kernel(uint4* __restrict__ p, int64_t n16) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = make_uint4(0, 0, 0, 0);
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

int stream_grid(int64_t items) {
  const int64_t need = (items + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  return static_cast<int>(need < 1 ? 1 : (need < cap ? need : cap));
}

inline size_t round_up256(size_t v) { return (v + 255) / 256 * 256; }
inline int64_t pad64(int64_t v) { return (v + 63) / 64 * 64; }

cudaError_t transpose(const mf_bf16* src, int64_t src_ld, const RunTable& rt, int64_t n_pad,
                      int64_t C, mf_bf16* dst, int64_t dst_ld, int32_t dst_col0,
                      cudaStream_t st) {
  if (n_pad == 0 || C == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(n_pad / kTile), static_cast<unsigned>(C / kTile));
  transpose_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint16_t*>(src), src_ld, rt,
                                         reinterpret_cast<uint16_t*>(dst), dst_ld, dst_col0);
  return cudaGetLastError();
}

// Each modality's tokens as runs of consecutive rows of the pack (a sample's
// image tokens, then its text tokens).
void modality_runs(const mf_sample_desc* desc, int32_t S, RunTable (&rt)[2]) {
  rt[0].n = rt[1].n = 0;
  int32_t row = 0, count[2] = {0, 0};
  for (int32_t s = 0; s < S; ++s) {
    const int32_t n[2] = {desc[s].frames * desc[s].grid_h * desc[s].grid_w, desc[s].n_text};
    for (int m = 0; m < 2; ++m) {
      if (n[m] > 0) {
        rt[m].src0[rt[m].n] = row;
        rt[m].dst0[rt[m].n] = count[m];
        ++rt[m].n;
        count[m] += n[m];
        row += n[m];
      }
    }
  }
  for (int m = 0; m < 2; ++m) rt[m].dst0[rt[m].n] = count[m];
}

}  // namespace

// Workspace of mf_mmdit_block_bwd, in the order the chain takes it.
struct BwdLayout {
  size_t row, wide, total;
  size_t x1, q, k, v, qr, kr, o, a, y1, x2, z, h, mlp, lse;
  size_t dmlp, dz, dx2, dy1, da, d_o, dqr, dkr, dv, dqkv, dx1;
  size_t wdownT, wupT, woT, wqkvT, yT, xT, attn_ws, ln_ws;
  BwdLayout(int32_t T, int32_t S, int32_t H, int32_t D, int32_t F) {
    const size_t hid = static_cast<size_t>(H) * D;
    row = round_up256(static_cast<size_t>(T) * hid * 2);
    wide = round_up256(static_cast<size_t>(T) * F * 2);
    const size_t tp = static_cast<size_t>(pad64(T));
    size_t p = 0;
    auto take = [&](size_t b) { const size_t at = p; p += round_up256(b); return at; };
    x1 = take(row); q = take(row); k = take(row); v = take(row); qr = take(row); kr = take(row);
    o = take(row); a = take(row); y1 = take(row); x2 = take(row); z = take(wide); h = take(wide);
    mlp = take(row); lse = take(static_cast<size_t>(H) * T * 4);
    dmlp = take(row); dz = take(wide); dx2 = take(row); dy1 = take(row); da = take(row);
    d_o = take(row); dqr = take(row); dkr = take(row); dv = take(row); dqkv = take(3 * row);
    dx1 = take(row);
    wdownT = take(2 * hid * F * 2); wupT = take(2 * hid * F * 2); woT = take(2 * hid * hid * 2);
    wqkvT = take(2 * hid * 3 * hid * 2);
    const size_t big = static_cast<size_t>(F) > 3 * hid ? static_cast<size_t>(F) : 3 * hid;
    yT = take(big * tp * 2); xT = take(big * tp * 2);
    attn_ws = take(mf_attn_bwd_workspace_size(T, S, H, D));
    ln_ws = take(mf_adaln_bwd_workspace_size(T));
    total = p + 256;
  }
};

}  // namespace mf

extern "C" {

size_t mf_mmdit_bwd_workspace_size(int32_t T, int32_t S, int32_t H, int32_t D, int32_t F) {
  if (T < 0 || S < 1 || H < 1 || D < 1 || F < 1) return 0;
  return mf::BwdLayout(T, S, H, D, F).total;
}

mf_status mf_mmdit_block_bwd(const mf_bf16* dy, const mf_bf16* x, const mf_bf16* Wq,
                             const mf_bf16* Wk, const mf_bf16* Wv, const mf_bf16* Wo,
                             const mf_bf16* Wup, const mf_bf16* Wdown, const float* mod_attn,
                             const float* mod_mlp, const mf_sample_desc* desc,
                             const int32_t* cu_seqlens_d, const int32_t* cu_seqlens_h,
                             const int32_t* pos_ids, const int32_t* tok_sample,
                             const uint8_t* tok_mod, int32_t S, int32_t H, int32_t D, int32_t F,
                             int32_t rope_axes, float base, float eps, mf_bf16* dx, mf_bf16* dWq,
                             mf_bf16* dWk, mf_bf16* dWv, mf_bf16* dWo, mf_bf16* dWup,
                             mf_bf16* dWdown, float* dmod_attn, float* dmod_mlp,
                             void* workspace, size_t ws_bytes, cudaStream_t stream) {
  using namespace mf;
  if (desc == nullptr || cu_seqlens_h == nullptr || S < 1 || S > MF_MAX_SAMPLES || H < 1 ||
      D < 1 || F < 256 || F % 256 != 0 || F > (1 << 20))
    return MF_ERR_INVALID;
  const int32_t hid = H * D;
  if (hid % 256 != 0) return MF_ERR_UNSUPPORTED;
  int32_t T = 0;
  if (!check_offsets(cu_seqlens_h, S, &T)) return MF_ERR_INVALID;
  // the weight-gradient products run over F (or hid) rows as one job table, and
  // the forward's over T rows: both within the linear layer's job limit
  if (static_cast<int64_t>(F) > static_cast<int64_t>(kMaxGemmTiles) * 128 ||
      static_cast<int64_t>(T) > static_cast<int64_t>(kMaxGemmTiles) * 128)
    return MF_ERR_UNSUPPORTED;
  for (int32_t s = 0; s < S; ++s) {
    const mf_sample_desc& d = desc[s];
    if (d.frames < 0 || d.grid_h < 0 || d.grid_w < 0 || d.n_text < 0 ||
        static_cast<int64_t>(d.frames) * d.grid_h * d.grid_w + d.n_text !=
            cu_seqlens_h[s + 1] - cu_seqlens_h[s])
      return MF_ERR_INVALID;
  }
  if (T == 0) return MF_OK;
  const BwdLayout L(T, S, H, D, F);
  const void* ins[] = {dy, x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp};
  mf_bf16* outs_bf[] = {dx, dWq, dWk, dWv, dWo, dWup, dWdown};
  for (const void* p : ins)
    if (p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) != 0) return MF_ERR_INVALID;
  for (const void* p : outs_bf)
    if (p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) != 0) return MF_ERR_INVALID;
  if (dmod_attn == nullptr || dmod_mlp == nullptr || workspace == nullptr ||
      (reinterpret_cast<uintptr_t>(dmod_attn) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(dmod_mlp) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0 || ws_bytes < L.total)
    return MF_ERR_INVALID;
  // every output is disjoint from every input, from the other outputs and from
  // the workspace
  const size_t rowb = static_cast<size_t>(T) * hid * 2;
  const size_t hh = static_cast<size_t>(hid) * hid * 2 * 2, hf = static_cast<size_t>(hid) * F * 2 * 2;
  const size_t modb = static_cast<size_t>(S) * 6 * hid * 4;
  const void* all_p[] = {dy, x, Wq, Wk, Wv, Wo, Wup, Wdown, mod_attn, mod_mlp, workspace,
                         dx, dWq, dWk, dWv, dWo, dWup, dWdown, dmod_attn, dmod_mlp};
  const size_t all_n[] = {rowb, rowb, hh, hh, hh, hh, hf, hf, modb, modb, ws_bytes,
                          rowb, hh, hh, hh, hh, hf, hf, modb, modb};
  constexpr int kIns = 11;
  for (int i = kIns; i < 20; ++i)
    for (int j = 0; j < 20; ++j) {
      if (i == j) continue;
      const uintptr_t a = reinterpret_cast<uintptr_t>(all_p[i]), b = reinterpret_cast<uintptr_t>(all_p[j]);
      if (a < b + all_n[j] && b < a + all_n[i]) return MF_ERR_INVALID;
    }
  KernelCtl ctl;
  if (cudaError_t ge = get_ctl(&ctl); ge != cudaSuccess) return MF_ERR_CUDA;
  bool pair = false;
  if (!linear_cta_pair(&pair)) return MF_ERR_CUDA;

  const uintptr_t w0 = (reinterpret_cast<uintptr_t>(workspace) + 255) / 256 * 256;
  auto bf = [&](size_t off) { return reinterpret_cast<mf_bf16*>(w0 + off); };
  mf_bf16 *x1 = bf(L.x1), *q = bf(L.q), *k = bf(L.k), *v = bf(L.v), *qr = bf(L.qr), *kr = bf(L.kr);
  mf_bf16 *o = bf(L.o), *a = bf(L.a), *y1 = bf(L.y1), *x2 = bf(L.x2), *z = bf(L.z), *h = bf(L.h);
  mf_bf16 *mlp = bf(L.mlp), *dmlp = bf(L.dmlp), *dz = bf(L.dz), *dx2 = bf(L.dx2), *dy1 = bf(L.dy1);
  mf_bf16 *da = bf(L.da), *d_o = bf(L.d_o), *dqr = bf(L.dqr), *dkr = bf(L.dkr), *dv = bf(L.dv);
  mf_bf16 *dqkv = bf(L.dqkv), *dx1 = bf(L.dx1);
  mf_bf16 *wdownT = bf(L.wdownT), *wupT = bf(L.wupT), *woT = bf(L.woT), *wqkvT = bf(L.wqkvT);
  mf_bf16 *yT = bf(L.yT), *xT = bf(L.xT);
  float* lse = reinterpret_cast<float*>(w0 + L.lse);
  void* attn_ws = reinterpret_cast<void*>(w0 + L.attn_ws);
  void* ln_ws = reinterpret_cast<void*>(w0 + L.ln_ws);
  const size_t attn_ws_bytes = mf_attn_bwd_workspace_size(T, S, H, D);
  const size_t ln_ws_bytes = mf_adaln_bwd_workspace_size(T);
  const float scale = 1.0f / std::sqrt(static_cast<float>(D));

  mf_status st;
  cudaError_t ce;
#define MF_STEP(call)          \
  st = (call);                 \
  if (st != MF_OK) return st;
#define MF_CUDA(call)                          \
  ce = (call);                                 \
  if (ce != cudaSuccess) return MF_ERR_CUDA;

  // ---- forward, keeping what the backward needs (bf16, as the forward stores it)
  MF_STEP(mf_adaln_modulate(x, mod_attn, tok_sample, tok_mod, T, S, hid, eps, x1, stream));
  MF_STEP(mf_modality_linear(x1, Wq, tok_mod, desc, S, hid, hid, MF_ACT_NONE, q, stream));
  MF_STEP(mf_modality_linear(x1, Wk, tok_mod, desc, S, hid, hid, MF_ACT_NONE, k, stream));
  MF_STEP(mf_modality_linear(x1, Wv, tok_mod, desc, S, hid, hid, MF_ACT_NONE, v, stream));
  MF_STEP(mf_rope_apply(q, k, pos_ids, T, H, D, rope_axes, base, qr, kr, stream));
  MF_STEP(mf_varlen_attn_fwd(qr, kr, v, cu_seqlens_d, cu_seqlens_h, S, H, D, scale, nullptr,
                             rope_axes, base, o, lse, nullptr, 0, stream));
  MF_STEP(mf_modality_linear(o, Wo, tok_mod, desc, S, hid, hid, MF_ACT_NONE, a, stream));
  MF_STEP(mf_gated_residual(x, a, mod_attn, tok_sample, tok_mod, T, S, hid, y1, stream));
  MF_STEP(mf_adaln_modulate(y1, mod_mlp, tok_sample, tok_mod, T, S, hid, eps, x2, stream));
  MF_STEP(mf_modality_linear(x2, Wup, tok_mod, desc, S, hid, F, MF_ACT_NONE, z, stream));
  const int64_t wide8 = static_cast<int64_t>(T) * F / 8;
  gelu_kernel<<<stream_grid(wide8), 256, 0, stream>>>(reinterpret_cast<const uint4*>(z), wide8,
                                                      reinterpret_cast<uint4*>(h));
  MF_CUDA(cudaGetLastError());
  MF_STEP(mf_modality_linear(h, Wdown, tok_mod, desc, S, F, hid, MF_ACT_NONE, mlp, stream));

  // ---- transposed weights, W[m] [N][K] -> W[m]^T [K][N] (the input gradients' products)
  RunTable ident;
  auto transpose_weights = [&](const mf_bf16* W, int32_t N, int32_t K, mf_bf16* WT, int64_t ld,
                               int32_t col0) -> cudaError_t {
    ident.n = 1;
    ident.src0[0] = 0;
    ident.dst0[0] = 0;
    ident.dst0[1] = N;
    for (int m = 0; m < 2; ++m) {
      const cudaError_t e = transpose(W + static_cast<size_t>(m) * N * K, K, ident, N, K,
                                      WT + static_cast<size_t>(m) * K * ld, ld, col0, stream);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  };
  MF_CUDA(transpose_weights(Wdown, hid, F, wdownT, hid, 0));  // [2][F][hid]
  MF_CUDA(transpose_weights(Wup, F, hid, wupT, F, 0));        // [2][hid][F]
  MF_CUDA(transpose_weights(Wo, hid, hid, woT, hid, 0));      // [2][hid][hid]
  MF_CUDA(transpose_weights(Wq, hid, hid, wqkvT, 3 * hid, 0));  // [2][hid][3 hid]
  MF_CUDA(transpose_weights(Wk, hid, hid, wqkvT, 3 * hid, hid));
  MF_CUDA(transpose_weights(Wv, hid, hid, wqkvT, 3 * hid, 2 * hid));

  // ---- MLP branch
  MF_STEP(mf_gated_residual_bwd(dy, mlp, mod_mlp, tok_sample, tok_mod, T, S, hid, dmlp, dmod_mlp,
                                stream));
  MF_STEP(mf_modality_linear(dmlp, wdownT, tok_mod, desc, S, hid, F, MF_ACT_NONE, dz, stream));
  gelu_bwd_kernel<<<stream_grid(wide8), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(z), reinterpret_cast<const uint4*>(dz), wide8,
      reinterpret_cast<uint4*>(dz));
  MF_CUDA(cudaGetLastError());
  MF_STEP(mf_modality_linear(dz, wupT, tok_mod, desc, S, F, hid, MF_ACT_NONE, dx2, stream));
  MF_STEP(mf_adaln_modulate_bwd(dx2, y1, mod_mlp, tok_sample, tok_mod, dy, T, S, hid, eps, dy1,
                                dmod_mlp, ln_ws, ln_ws_bytes, stream));
  // ---- attention branch
  MF_STEP(mf_gated_residual_bwd(dy1, a, mod_attn, tok_sample, tok_mod, T, S, hid, da, dmod_attn,
                                stream));
  MF_STEP(mf_modality_linear(da, woT, tok_mod, desc, S, hid, hid, MF_ACT_NONE, d_o, stream));
  MF_STEP(mf_varlen_attn_bwd(qr, kr, v, o, d_o, lse, cu_seqlens_d, cu_seqlens_h, S, H, D, scale,
                             dqr, dkr, dv, attn_ws, attn_ws_bytes, stream));
  MF_STEP(mf_rope_bwd(dqr, dkr, pos_ids, T, H, D, rope_axes, base, dqr, dkr, stream));
  const int64_t row8 = static_cast<int64_t>(T) * hid / 8;
  pack3_kernel<<<stream_grid(row8), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(dqr), reinterpret_cast<const uint4*>(dkr),
      reinterpret_cast<const uint4*>(dv), T, hid / 8, reinterpret_cast<uint4*>(dqkv));
  MF_CUDA(cudaGetLastError());
  MF_STEP(mf_modality_linear(dqkv, wqkvT, tok_mod, desc, S, 3 * hid, hid, MF_ACT_NONE, dx1,
                             stream));
  MF_STEP(mf_adaln_modulate_bwd(dx1, x, mod_attn, tok_sample, tok_mod, dy1, T, S, hid, eps, dx,
                                dmod_attn, ln_ws, ln_ws_bytes, stream));

  // ---- weight gradients: dW[m] = d_out_m^T in_m over the modality's tokens
  RunTable runs[2];
  modality_runs(desc, S, runs);
  struct WGrad {
    const mf_bf16* d_out;  // [T][N], row stride ld_out
    int64_t ld_out;
    const mf_bf16* in;     // [T][K]
    int32_t N, K;
    mf_bf16* dW;           // [2][N][K]
  };
  const WGrad grads[] = {
      {dmlp, hid, h, hid, F, dWdown}, {dz, F, x2, F, hid, dWup},
      {da, hid, o, hid, hid, dWo},    {dqkv, 3 * hid, x1, hid, hid, dWq},
      {dqkv + hid, 3 * hid, x1, hid, hid, dWk}, {dqkv + 2 * hid, 3 * hid, x1, hid, hid, dWv}};
  for (int m = 0; m < 2; ++m) {
    const int64_t tm = runs[m].dst0[runs[m].n];
    const int64_t tp = pad64(tm);
    const mf_bf16* last_in = nullptr;
    for (const WGrad& g : grads) {
      mf_bf16* out = g.dW + static_cast<size_t>(m) * g.N * g.K;
      if (tm == 0) {
        const int64_t n16 = static_cast<int64_t>(g.N) * g.K / 8;
        zero_kernel<<<stream_grid(n16), 256, 0, stream>>>(reinterpret_cast<uint4*>(out), n16);
        MF_CUDA(cudaGetLastError());
        continue;
      }
      if (g.in != last_in) {  // in_m^T [K][tp], shared by the three input projections
        MF_CUDA(transpose(g.in, g.K, runs[m], tp, g.K, xT, tp, 0, stream));
        last_in = g.in;
      }
      MF_CUDA(transpose(g.d_out, g.ld_out, runs[m], tp, g.N, yT, tp, 0, stream));
      MF_CUDA(launch_linear_plain(yT, xT, g.N, static_cast<int32_t>(tp), g.K, pair, out, ctl,
                                  stream));
    }
  }
#undef MF_CUDA
#undef MF_STEP
  return MF_OK;
}

}  // extern "C"
