// elementwise.cu -- the HBM-bound steps of the packed joint-attention block on
// sm_100a: pack ids, adaLN modulation vectors, modality-specific adaLN, per-
// sample RoPE and the standalone gated residual. Every kernel moves 16-byte
// vectors, rows are reduced with warp shuffles, and grids are sized in multiples
// of the SM count with grid-stride loops.
//
// Sources (page title, section): picx.dev "Mage-Flow" summary, Methodology >
// Native-Resolution MMDiT (packing, modality-specific normalization, 3D RoPE for
// edits) and > Training Infrastructure (fused adaptive normalization / RoPE /
// gating); gist.science "Resumo Tecnico: Mage-Flow", Metodologia > 2. NR-MMDiT
// (per-sample 2D rotary embeddings).
#include <cuda_bf16.h>

#include <cmath>
#include <cstdint>

#include "cfg_internal.h"
#include "mf_internal.h"
#include "mf_ptx.cuh"

namespace mf {

namespace {

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

inline int grid_for(long long work_items, int threads, int max_blocks_per_sm) {
  long long need = (work_items + threads - 1) / threads;
  long long cap = static_cast<long long>(sm_count()) * max_blocks_per_sm;
  if (need < 1) need = 1;
  return static_cast<int>(need < cap ? need : cap);
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
  uint4 u;
  u.x = pack_bf16x2(f[0], f[1]);
  u.y = pack_bf16x2(f[2], f[3]);
  u.z = pack_bf16x2(f[4], f[5]);
  u.w = pack_bf16x2(f[6], f[7]);
  return u;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ------------------------------------------------------------ pack ids
__global__ void __launch_bounds__(256) pack_ids_kernel(const PackParams p, int32_t* cu_d,
                                                       int32_t* pos, int32_t* tok_sample,
                                                       uint8_t* tok_mod) {
  __shared__ int32_t s_cu[MF_MAX_SAMPLES + 1];
  for (int i = threadIdx.x; i <= p.S; i += blockDim.x) s_cu[i] = p.cu[i];
  __syncthreads();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i <= p.S; i += blockDim.x) cu_d[i] = s_cu[i];
  const int stride = gridDim.x * blockDim.x;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < p.T; t += stride) {
    // sample of token t: the largest s with cu[s] <= t (empty samples skipped)
    int lo = 0, hi = p.S - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int s = lo;
    const int i = t - s_cu[s];
    const int gh = p.grid_h[s], gw = p.grid_w[s];
    const int plane = gh * gw;
    const int n_img = p.frames[s] * plane;
    int f, h, w, m;
    if (i < n_img) {
      f = i / plane;
      const int r = i - f * plane;
      h = r / gw;
      w = r - h * gw;
      m = 0;
    } else {
      const int q = (gh > gw ? gh : gw) + (i - n_img);
      f = h = w = q;
      m = 1;
    }
    pos[3 * t + 0] = f;
    pos[3 * t + 1] = h;
    pos[3 * t + 2] = w;
    tok_sample[t] = s;
    tok_mod[t] = static_cast<uint8_t>(m);
  }
}

// ------------------------------------------------------------ adaLN params
// mod[s][n] = sum_c c[s][c] * W[c][n], n in [0, 6*hid). A 256-thread CTA covers
// 128 columns: 32 threads read float4 column groups, 8 warps split the
// conditioning dimension into slices, and the slice sums meet in shared memory
// in a fixed order (the result does not depend on scheduling). Eight samples
// per pass share each W load.
constexpr int kParamSamples = 8;
constexpr int kMaxCond = 1024;
constexpr int kParamSlices = 8;
constexpr int kParamCols4 = 32;  // float4 column groups per CTA

__global__ void __launch_bounds__(256) adaln_params_kernel(const float* __restrict__ c,
                                                           const float4* __restrict__ W4, int S,
                                                           int C, int N4, float4* __restrict__ mod4) {
  // the conditioning rows and, after them, the slice partial sums share one
  // 32 KB buffer
  __shared__ __align__(16) unsigned char buf[kParamSamples * kMaxCond * 4];
  static_assert(sizeof(float4) * kParamSlices * kParamSamples * kParamCols4 <= sizeof(buf), "");
  auto s_c = reinterpret_cast<float(*)[kMaxCond]>(buf);
  auto s_part = reinterpret_cast<float4(*)[kParamSamples][kParamCols4]>(buf);
  const int g = threadIdx.x & 31;      // column group inside the CTA
  const int slice = threadIdx.x >> 5;  // slice of the conditioning dimension
  const int n4 = blockIdx.x * kParamCols4 + g;
  const int per_slice = (C + kParamSlices - 1) / kParamSlices;
  const int c0 = slice * per_slice;
  const int c1 = min(C, c0 + per_slice);
  for (int s0 = 0; s0 < S; s0 += kParamSamples) {
    const int ns = min(kParamSamples, S - s0);
    __syncthreads();
    for (int i = threadIdx.x; i < ns * C; i += blockDim.x)
      s_c[i / C][i % C] = c[static_cast<size_t>(s0 + i / C) * C + (i % C)];
    __syncthreads();
    float4 acc[kParamSamples];
#pragma unroll
    for (int u = 0; u < kParamSamples; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (n4 < N4) {
#pragma unroll 4
      for (int cc = c0; cc < c1; ++cc) {
        const float4 w = __ldg(W4 + static_cast<size_t>(cc) * N4 + n4);
#pragma unroll
        for (int u = 0; u < kParamSamples; ++u) {
          const float cv = s_c[u][cc];
          acc[u].x = fmaf(cv, w.x, acc[u].x);
          acc[u].y = fmaf(cv, w.y, acc[u].y);
          acc[u].z = fmaf(cv, w.z, acc[u].z);
          acc[u].w = fmaf(cv, w.w, acc[u].w);
        }
      }
    }
    __syncthreads();  // every thread is done with s_c
#pragma unroll
    for (int u = 0; u < kParamSamples; ++u) s_part[slice][u][g] = acc[u];
    __syncthreads();
    for (int i = threadIdx.x; i < ns * kParamCols4; i += blockDim.x) {
      const int u = i / kParamCols4, gg = i % kParamCols4;
      const int nn4 = blockIdx.x * kParamCols4 + gg;
      if (nn4 < N4) {
        float4 v = s_part[0][u][gg];
#pragma unroll
        for (int sl = 1; sl < kParamSlices; ++sl) {
          const float4 q = s_part[sl][u][gg];
          v.x += q.x; v.y += q.y; v.z += q.z; v.w += q.w;
        }
        mod4[static_cast<size_t>(s0 + u) * N4 + nn4] = v;
      }
    }
  }
}

// ------------------------------------------------------------ adaLN modulate
// One warp per token row; the row stays in registers as packed bf16 (NCH
// 16-byte chunks per lane) across the mean pass, the variance pass and the
// output pass. Each CTA takes a contiguous range of rows (its warps
// interleaved inside it), so the rows an SM works on at a time mostly share a
// sample and modality and their shift / scale vectors stay in L1.
// The register cap (up to three 256-thread CTAs per SM) keeps enough
// rows in flight to cover HBM latency.
template <int NCH>
__global__ void __launch_bounds__(256, (NCH <= 4 ? 3 : (NCH <= 12 ? 2 : 1))) adaln_modulate_kernel(
    const uint4* __restrict__ x, const float* __restrict__ mod,
    const int32_t* __restrict__ tok_sample, const uint8_t* __restrict__ tok_mod, int T, int S,
    int hid, float eps, uint4* __restrict__ x_mod, KernelCtl ctl) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int nchunk = hid >> 3;
  const float inv_hid = 1.f / static_cast<float>(hid);
  const int per_block = (T + gridDim.x - 1) / gridDim.x;
  const int row_end = min(T, (blockIdx.x + 1) * per_block);
  for (int row = blockIdx.x * per_block + (threadIdx.x >> 5); row < row_end; row += wpb) {
    const int s = __ldg(tok_sample + row);
    const int m = __ldg(tok_mod + row);
    if (s < 0 || s >= S || m > 1) {
      if (lane == 0) atomicCAS(ctl.err, 0, static_cast<int>(MF_ERR_INVALID));
      continue;
    }
    const uint4* xr = x + static_cast<size_t>(row) * nchunk;
    uint4 v[NCH];
#pragma unroll
    for (int u = 0; u < NCH; ++u) {
      const int idx = lane + 32 * u;
      if (idx < nchunk) v[u] = __ldcs(xr + idx);
      else v[u] = make_uint4(0, 0, 0, 0);
    }
    float sum = 0.f;
#pragma unroll
    for (int u = 0; u < NCH; ++u) {
      float f[8];
      unpack8(v[u], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) sum += f[e];
    }
    const float mean = warp_sum(sum) * inv_hid;
    float sq = 0.f;
#pragma unroll
    for (int u = 0; u < NCH; ++u) {
      if (lane + 32 * u < nchunk) {
        float f[8];
        unpack8(v[u], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float d = f[e] - mean;
          sq = fmaf(d, d, sq);
        }
      }
    }
    const float rstd = rsqrtf(warp_sum(sq) * inv_hid + eps);
    const float* shift = mod + (static_cast<size_t>(s) * 2 + m) * 3 * hid;
    const float* scale = shift + hid;
    uint4* orow = x_mod + static_cast<size_t>(row) * nchunk;
#pragma unroll
    for (int u = 0; u < NCH; ++u) {
      const int idx = lane + 32 * u;
      if (idx < nchunk) {
        float f[8];
        unpack8(v[u], f);
        const float4 sh0 = __ldg(reinterpret_cast<const float4*>(shift + idx * 8));
        const float4 sh1 = __ldg(reinterpret_cast<const float4*>(shift + idx * 8 + 4));
        const float4 sc0 = __ldg(reinterpret_cast<const float4*>(scale + idx * 8));
        const float4 sc1 = __ldg(reinterpret_cast<const float4*>(scale + idx * 8 + 4));
        const float shv[8] = {sh0.x, sh0.y, sh0.z, sh0.w, sh1.x, sh1.y, sh1.z, sh1.w};
        const float scv[8] = {sc0.x, sc0.y, sc0.z, sc0.w, sc1.x, sc1.y, sc1.z, sc1.w};
        float out[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) out[e] = fmaf((f[e] - mean) * rstd, 1.f + scv[e], shv[e]);
        __stcs(orow + idx, pack8(out));
      }
    }
  }
}

// ------------------------------------------------------------ packed CFG combine
// One thread per 16-byte chunk of output rows (grid-stride): the chunk's pair by
// binary search of the row map in the kernel parameters, then out = fma(w,
// c - u, u) in fp32 on the two branches' chunks (picx.dev "Mage-Flow" summary,
// Methodology > NR-MMDiT, "Packed CFG inference"; the combine is the usual
// classifier-free guidance form).
__global__ void __launch_bounds__(256) cfg_combine_kernel(const uint4* __restrict__ v,
                                                          const CfgTable tab, int C, float w,
                                                          uint4* __restrict__ out) {
  const int cpr = C >> 3;  // chunks per row
  const long long total = static_cast<long long>(tab.out0[tab.P]) * cpr;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long gi = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; gi < total;
       gi += stride) {
    const int r = static_cast<int>(gi / cpr);
    const int c = static_cast<int>(gi - static_cast<long long>(r) * cpr);
    int lo = 0, hi = tab.P - 1;  // last pair with out0[p] <= r
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tab.out0[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int i = r - tab.out0[lo];
    float fc[8], fu[8], o[8];
    unpack8(__ldcs(v + static_cast<size_t>(tab.cond0[lo] + i) * cpr + c), fc);
    unpack8(__ldcs(v + static_cast<size_t>(tab.uncond0[lo] + i) * cpr + c), fu);
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = fmaf(w, fc[e] - fu[e], fu[e]);
    __stcs(out + gi, pack8(o));
  }
}

// ------------------------------------------------------------ RoPE
// One thread per (token, 8-channel chunk): it computes the four pair angles of
// its chunk once and applies them to that chunk of every head of q and k.
// q_out / k_out may alias q / k: each element is read before it is written by
// the same thread, so the pointers carry no __restrict__.
__global__ void __launch_bounds__(256) rope_kernel(const uint4* q, const uint4* k,
                                                   const int32_t* __restrict__ pos, int T, int H,
                                                   int D, const RopeTable tab, uint4* q_out,
                                                   uint4* k_out) {
  const int cpr = D >> 3;  // chunks per head row
  const long long total = static_cast<long long>(T) * cpr;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long gi = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; gi < total;
       gi += stride) {
    const int t = static_cast<int>(gi / cpr);
    const int cch = static_cast<int>(gi - static_cast<long long>(t) * cpr);
    float cs[4], sn[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int pr = cch * 4 + j;
      const int comp = tab.comp[pr];
      if (comp >= 0) {
        const float theta = static_cast<float>(__ldg(pos + 3 * t + comp)) * tab.inv_freq[pr];
        sincosf(theta, &sn[j], &cs[j]);
      } else {
        cs[j] = 1.f;
        sn[j] = 0.f;
      }
    }
    // four heads per step: 8 independent 16-byte loads in flight per thread
#pragma unroll 4
    for (int h = 0; h < H; ++h) {
      const size_t off = (static_cast<size_t>(t) * H + h) * cpr + cch;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint4* src = which ? k : q;
        uint4* dst = which ? k_out : q_out;
        if (src == nullptr) continue;
        float f[8], o[8];
        unpack8(__ldcs(src + off), f);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          o[2 * j] = f[2 * j] * cs[j] - f[2 * j + 1] * sn[j];
          o[2 * j + 1] = f[2 * j] * sn[j] + f[2 * j + 1] * cs[j];
        }
        __stcs(dst + off, pack8(o));
      }
    }
  }
}

// ------------------------------------------------------------ gated residual
// y may alias x (in-place residual), so x and y carry no __restrict__.
__global__ void __launch_bounds__(256) gated_residual_kernel(
    const uint4* x, const uint4* __restrict__ o, const float* __restrict__ mod,
    const int32_t* __restrict__ tok_sample, const uint8_t* __restrict__ tok_mod, int T, int S,
    int hid, uint4* y, KernelCtl ctl) {
  const int cpr = hid >> 3;
  const long long total = static_cast<long long>(T) * cpr;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long gi = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; gi < total;
       gi += stride) {
    const int t = static_cast<int>(gi / cpr);
    const int cch = static_cast<int>(gi - static_cast<long long>(t) * cpr);
    const int s = __ldg(tok_sample + t);
    const int m = __ldg(tok_mod + t);
    if (s < 0 || s >= S || m > 1) {
      atomicCAS(ctl.err, 0, static_cast<int>(MF_ERR_INVALID));
      continue;
    }
    const float* gate = mod + ((static_cast<size_t>(s) * 2 + m) * 3 + 2) * hid + cch * 8;
    const float4 g0 = __ldg(reinterpret_cast<const float4*>(gate));
    const float4 g1 = __ldg(reinterpret_cast<const float4*>(gate + 4));
    const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    float xf[8], of[8], out[8];
    unpack8(x[gi], xf);
    unpack8(__ldcs(o + gi), of);
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = fmaf(gv[e], of[e], xf[e]);
    __stcs(y + gi, pack8(out));
  }
}

__global__ void selftest_wait_kernel(KernelCtl ctl) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the wait runs out after ctl.wait_limit_ns,
  // records MF_ERR_TIMEOUT and returns.
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, ctl, &abort_flag);
  __syncthreads();
}

// Pairs (2i, 2i+1) through exp2_poly2, as the attention softmax uses it; a
// trailing odd element is paired with itself.
__global__ void selftest_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i < n) {
    const float a = x[i];
    const float b = (i + 1 < n) ? x[i + 1] : a;
    float pa, pb;
    exp2_poly2(a, b, pa, pb);
    y[i] = pa;
    if (i + 1 < n) y[i + 1] = pb;
  }
}

}  // namespace

cudaError_t launch_selftest_exp2(const float* x, float* y, int32_t n, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  selftest_exp2_kernel<<<(n / 2 + 256) / 256, 256, 0, st>>>(x, y, n);
  return cudaGetLastError();
}

// ------------------------------------------------------------ launchers
cudaError_t launch_pack_ids(const PackParams& p, int32_t* cu_d, int32_t* pos,
                            int32_t* tok_sample, uint8_t* tok_mod, cudaStream_t st) {
  const int grid = grid_for(p.T > 0 ? p.T : 1, 256, 8);
  pack_ids_kernel<<<grid, 256, 0, st>>>(p, cu_d, pos, tok_sample, tok_mod);
  return cudaGetLastError();
}

cudaError_t launch_adaln_params(const float* c, const float* W, int32_t S, int32_t C,
                                int32_t hid, float* mod, cudaStream_t st) {
  const int N4 = 6 * hid / 4;  // hid % 8 == 0, so whole float4 groups
  adaln_params_kernel<<<(N4 + kParamCols4 - 1) / kParamCols4, 256, 0, st>>>(
      c, reinterpret_cast<const float4*>(W), S, C, N4, reinterpret_cast<float4*>(mod));
  return cudaGetLastError();
}

cudaError_t launch_adaln_modulate(const mf_bf16* x, const float* mod, const int32_t* tok_sample,
                                  const uint8_t* tok_mod, int32_t T, int32_t S, int32_t hid,
                                  float eps, mf_bf16* x_mod, const KernelCtl& ctl,
                                  cudaStream_t st) {
  const int nchunk = hid / 8;
  const int per_lane = (nchunk + 31) / 32;
  // resident CTAs only (persistent): 3, 2 or 1 per SM by the register cap
  const int per_sm = per_lane <= 4 ? 3 : (per_lane <= 12 ? 2 : 1);
  const int grid = grid_for(static_cast<long long>(T) * 32, 256, per_sm);
  auto X = reinterpret_cast<const uint4*>(x);
  auto XM = reinterpret_cast<uint4*>(x_mod);
#define MF_ADALN_CASE(N)                                                                   \
  if (per_lane <= N) {                                                                     \
    adaln_modulate_kernel<N><<<grid, 256, 0, st>>>(X, mod, tok_sample, tok_mod, T, S, hid, \
                                                   eps, XM, ctl);                          \
    return cudaGetLastError();                                                             \
  }
  MF_ADALN_CASE(1)
  MF_ADALN_CASE(2)
  MF_ADALN_CASE(4)
  MF_ADALN_CASE(8)
  MF_ADALN_CASE(12)
  MF_ADALN_CASE(16)
#undef MF_ADALN_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_rope(const mf_bf16* q, const mf_bf16* k, const int32_t* pos_ids, int32_t T,
                        int32_t H, int32_t D, const RopeTable& tab, mf_bf16* q_out,
                        mf_bf16* k_out, cudaStream_t st) {
  const long long work = static_cast<long long>(T) * (D / 8);
  const int grid = grid_for(work, 256, 8);
  rope_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(q),
                                    reinterpret_cast<const uint4*>(k), pos_ids, T, H, D, tab,
                                    reinterpret_cast<uint4*>(q_out),
                                    reinterpret_cast<uint4*>(k_out));
  return cudaGetLastError();
}

cudaError_t launch_gated_residual(const mf_bf16* x, const mf_bf16* o, const float* mod,
                                  const int32_t* tok_sample, const uint8_t* tok_mod, int32_t T,
                                  int32_t S, int32_t hid, mf_bf16* y, const KernelCtl& ctl,
                                  cudaStream_t st) {
  const long long work = static_cast<long long>(T) * (hid / 8);
  const int grid = grid_for(work, 256, 8);
  gated_residual_kernel<<<grid, 256, 0, st>>>(
      reinterpret_cast<const uint4*>(x), reinterpret_cast<const uint4*>(o), mod, tok_sample,
      tok_mod, T, S, hid, reinterpret_cast<uint4*>(y), ctl);
  return cudaGetLastError();
}

cudaError_t launch_cfg_combine(const mf_bf16* v, const CfgTable& tab, int32_t C, float w,
                               mf_bf16* out, cudaStream_t st) {
  const long long work = static_cast<long long>(tab.out0[tab.P]) * (C / 8);
  if (work == 0) return cudaSuccess;
  const int grid = grid_for(work, 256, 8);
  cfg_combine_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(v), tab, C, w,
                                           reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(uint64_t limit_ns, const KernelCtl& ctl, cudaStream_t st) {
  KernelCtl c = ctl;
  c.wait_limit_ns = limit_ns;
  selftest_wait_kernel<<<1, 32, 0, st>>>(c);
  return cudaGetLastError();
}

namespace {

// (cos, sin) of p * inv_freq[j] for every position p < P and pair column j <
// npa; the angle is the same fp32 product the RoPE pass forms.
__global__ void __launch_bounds__(256) rope_table_kernel(float2* __restrict__ tab, int P, int npa,
                                                         const RopeTable rt) {
  const long long n = static_cast<long long>(P) * npa;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(i / npa);
    const int j = static_cast<int>(i - static_cast<long long>(p) * npa);
    float sn, cs;
    sincosf(static_cast<float>(p) * rt.inv_freq[j], &sn, &cs);
    tab[i] = make_float2(cs, sn);
  }
}

}  // namespace

cudaError_t launch_rope_table(int32_t D, int32_t rope_axes, float base, int32_t P, void* tab,
                              AttnRopeParams* r, cudaStream_t st) {
  RopeTable rt;
  make_rope_table(D, rope_axes, base, &rt);
  const int npa = D / (2 * rope_axes);
  r->tab = tab;
  r->P = P;
  r->axes = rope_axes;
  const long long n = static_cast<long long>(P) * npa;
  if (n == 0) return cudaSuccess;
  const int grid = grid_for(n, 256, 4);
  rope_table_kernel<<<grid, 256, 0, st>>>(static_cast<float2*>(tab), P, npa, rt);
  return cudaGetLastError();
}

void make_rope_table(int32_t D, int32_t rope_axes, float base, RopeTable* tab) {
  const int d_a = 2 * (D / (2 * rope_axes));
  for (int p = 0; p < 64; ++p) {
    tab->inv_freq[p] = 0.f;
    tab->comp[p] = -1;
  }
  for (int p = 0; p < D / 2; ++p) {
    const int a = (2 * p) / d_a;
    if (a >= rope_axes) continue;
    const int i = p - a * (d_a / 2);
    tab->comp[p] = (rope_axes == 2) ? (a + 1) : a;
    tab->inv_freq[p] =
        static_cast<float>(std::pow(static_cast<double>(base), -2.0 * i / static_cast<double>(d_a)));
  }
}

}  // namespace mf
