// block_bwd.cu -- backward of the gated residual and of the modality-specific
// adaLN modulation (the HBM-bound steps of the block's backward).
//
// What it computes (picx.dev "Mage-Flow" summary, Methodology > Native-
// Resolution MMDiT: modality-specific adaptive normalization and gating;
// Training Infrastructure: the packed model is trained): with s the token's
// sample and m its modality,
//   y = x + gate[s,m] * O:
//     dO = gate[s,m] * dy,   dgate[s,m] = sum over the tokens of (s,m) of dy * O
//     (dx = dy is the caller's identity path);
//   x_mod = xhat * (1 + scale[s,m]) + shift[s,m], xhat = (x - mean) * rstd:
//     g = dx_mod * (1 + scale),  dx = resid + (g - mean(g) - xhat * mean(g * xhat)) * rstd,
//     dshift[s,m] = sum dx_mod,  dscale[s,m] = sum dx_mod * xhat.
//
// Kernels:
//   zero_mod_slots_kernel  zeroes the modulation-gradient slots a call writes.
//   gate_bwd_kernel        one thread per (64-row chunk, 8 channels): dO for its
//                          rows and the running sum of dy * O, flushed with fp32
//                          atomics whenever the (sample, modality) of the rows
//                          changes (rows of a pack are grouped by sample, image
//                          tokens before text, so a chunk meets few changes).
//   ln_bwd_rows_kernel     one warp per row: mean and rstd of x, then mean(g)
//                          and mean(g * xhat), then dx; writes (mean, rstd).
//   ln_bwd_cols_kernel     like gate_bwd_kernel, for dshift and dscale (reads
//                          x, dx_mod and the row statistics).
// 16-byte vector accesses throughout; bad sample / modality ids are recorded
// as MF_ERR_INVALID and their rows skipped.
//
// The modulation map mod = c W (no bias, no activation; [S][C] x [C][6 hid]) has
// the backward dW = c^T dmod and dc = dmod W^T:
//   params_dw_kernel       one thread per (4 columns, 16 rows of W): the S-term
//                          sums for its 16 x 4 outputs, samples in order.
//   params_dc_kernel       one CTA per conditioning channel: the dot products
//                          of W's row with every sample's dmod row, 16-byte
//                          loads, partial sums reduced in a fixed order.
// Neither uses atomics, so both are deterministic.
#include <cuda_bf16.h>

#include <cmath>
#include <cstdint>

#include "block_bwd_internal.h"
#include "mf_internal.h"
#include "mf_ptx.cuh"

namespace mf {

namespace {

constexpr int kRowsPerChunk = 64;
constexpr int kColThreads = 128;  // threads per CTA of the column kernels (8 channels each)

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

__device__ __forceinline__ void load8f(const float* p, float (&f)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p + 4));
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

__device__ __forceinline__ void atomic_add8(float* p, const float (&f)[8]) {
#pragma unroll
  for (int e = 0; e < 8; ++e) atomicAdd(p + e, f[e]);
}

// dmod[s][m][j][i] = 0 for every slot j whose bit is set in slot_mask.
__global__ void __launch_bounds__(256) zero_mod_slots_kernel(float* dmod, long long n, int hid,
                                                             int slot_mask) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>((i / hid) % 3);
    if ((slot_mask >> j) & 1) dmod[i] = 0.f;
  }
}

// Valid (sample, modality) of token t, or false (recorded) for a bad id.
__device__ __forceinline__ bool token_ids(const int32_t* tok_sample, const uint8_t* tok_mod,
                                          int t, int S, int& s, int& m, const KernelCtl& ctl) {
  s = __ldg(tok_sample + t);
  m = __ldg(tok_mod + t);
  if (s < 0 || s >= S || m > 1) {
    atomicCAS(ctl.err, 0, static_cast<int>(MF_ERR_INVALID));
    return false;
  }
  return true;
}

// Rows taken per step by the gate backward: their ids and data are all
// requested before any is used, so each thread keeps kColUnroll rows of loads
// in flight instead of one (0.67 -> 0.83 of HBM on the training pack; the
// same change slowed the adaLN column sums, 0.47 -> 0.42, so they keep one).
constexpr int kColUnroll = 4;

// grid: (row chunks, channel groups / kColThreads)
__global__ void __launch_bounds__(kColThreads) gate_bwd_kernel(
    const uint4* dy, const uint4* __restrict__ o, const float* __restrict__ mod,
    const int32_t* __restrict__ tok_sample, const uint8_t* __restrict__ tok_mod, int T, int S,
    int hid, uint4* d_o, float* __restrict__ dmod, KernelCtl ctl) {
  const int groups = hid >> 3;
  const int g = blockIdx.y * kColThreads + threadIdx.x;
  if (g >= groups) return;
  const int r0 = blockIdx.x * kRowsPerChunk;
  const int r1 = min(T, r0 + kRowsPerChunk);
  int cs = -1, cm = -1;  // (sample, modality) of the running sum
  float gate[8], acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) gate[e] = acc[e] = 0.f;
  for (int t0 = r0; t0 < r1; t0 += kColUnroll) {
    int s[kColUnroll], m[kColUnroll];
    bool ok[kColUnroll];
    uint4 vy[kColUnroll], vo[kColUnroll];
#pragma unroll
    for (int u = 0; u < kColUnroll; ++u) {
      const int t = t0 + u;
      ok[u] = t < r1 && token_ids(tok_sample, tok_mod, t, S, s[u], m[u], ctl);
      const size_t off = static_cast<size_t>(t < r1 ? t : r0) * groups + g;
      vy[u] = dy[off];
      vo[u] = __ldg(o + off);
    }
#pragma unroll
    for (int u = 0; u < kColUnroll; ++u) {
      if (!ok[u]) continue;
      if (s[u] != cs || m[u] != cm) {
        if (cs >= 0) atomic_add8(dmod + ((static_cast<size_t>(cs) * 2 + cm) * 3 + 2) * hid + 8 * g, acc);
        cs = s[u];
        cm = m[u];
        load8f(mod + ((static_cast<size_t>(cs) * 2 + cm) * 3 + 2) * hid + 8 * g, gate);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
      }
      float fy[8], fo[8], out[8];
      unpack8(vy[u], fy);
      unpack8(vo[u], fo);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        acc[e] = fmaf(fy[e], fo[e], acc[e]);
        out[e] = gate[e] * fy[e];
      }
      d_o[static_cast<size_t>(t0 + u) * groups + g] = pack8(out);
    }
  }
  if (cs >= 0) atomic_add8(dmod + ((static_cast<size_t>(cs) * 2 + cm) * 3 + 2) * hid + 8 * g, acc);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}

// One warp per row (grid-stride over rows, 8 warps per CTA). The row is read
// three times (statistics, the two means, the output); the second and third
// reads hit L1 / L2.
__global__ void __launch_bounds__(256) ln_bwd_rows_kernel(
    const uint4* __restrict__ dxm, const uint4* __restrict__ x, const uint4* resid,
    const float* __restrict__ mod, const int32_t* __restrict__ tok_sample,
    const uint8_t* __restrict__ tok_mod, int T, int S, int hid, float eps, uint4* dx,
    float2* __restrict__ stats, KernelCtl ctl) {
  const int lane = threadIdx.x & 31;
  const int groups = hid >> 3;
  const float inv_n = 1.f / static_cast<float>(hid);
  for (int t = blockIdx.x * 8 + (threadIdx.x >> 5); t < T; t += gridDim.x * 8) {
    int s, m;
    if (!token_ids(tok_sample, tok_mod, t, S, s, m, ctl)) continue;
    const uint4* xr = x + static_cast<size_t>(t) * groups;
    const uint4* gr = dxm + static_cast<size_t>(t) * groups;
    const float* scale = mod + ((static_cast<size_t>(s) * 2 + m) * 3 + 1) * hid;
    // mean and variance of x (two passes over the row for the variance)
    float sum = 0.f;
    for (int c = lane; c < groups; c += 32) {
      float f[8];
      unpack8(__ldg(xr + c), f);
#pragma unroll
      for (int e = 0; e < 8; ++e) sum += f[e];
    }
    const float mean = warp_sum(sum) * inv_n;
    float sq = 0.f;
    for (int c = lane; c < groups; c += 32) {
      float f[8];
      unpack8(__ldg(xr + c), f);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = f[e] - mean;
        sq = fmaf(d, d, sq);
      }
    }
    const float rstd = 1.f / sqrtf(warp_sum(sq) * inv_n + eps);
    // mean(g) and mean(g * xhat), g = dx_mod * (1 + scale)
    float sg = 0.f, sgx = 0.f;
    for (int c = lane; c < groups; c += 32) {
      float f[8], d[8], sc[8];
      unpack8(__ldg(xr + c), f);
      unpack8(__ldg(gr + c), d);
      load8f(scale + 8 * c, sc);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float gg = d[e] * (1.f + sc[e]);
        sg += gg;
        sgx = fmaf(gg, (f[e] - mean) * rstd, sgx);
      }
    }
    const float mg = warp_sum(sg) * inv_n;
    const float mgx = warp_sum(sgx) * inv_n;
    for (int c = lane; c < groups; c += 32) {
      float f[8], d[8], sc[8], r[8], out[8];
      unpack8(__ldg(xr + c), f);
      unpack8(__ldg(gr + c), d);
      load8f(scale + 8 * c, sc);
      const size_t off = static_cast<size_t>(t) * groups + c;
      if (resid != nullptr) {
        unpack8(resid[off], r);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float xh = (f[e] - mean) * rstd;
        const float gg = d[e] * (1.f + sc[e]);
        out[e] = r[e] + (gg - mg - xh * mgx) * rstd;
      }
      dx[off] = pack8(out);
    }
    if (lane == 0) stats[t] = make_float2(mean, rstd);
  }
}

// grid: (row chunks, channel groups / kColThreads)
__global__ void __launch_bounds__(kColThreads) ln_bwd_cols_kernel(
    const uint4* __restrict__ dxm, const uint4* __restrict__ x, const float2* __restrict__ stats,
    const int32_t* __restrict__ tok_sample, const uint8_t* __restrict__ tok_mod, int T, int S,
    int hid, float* __restrict__ dmod, KernelCtl ctl) {
  const int groups = hid >> 3;
  const int g = blockIdx.y * kColThreads + threadIdx.x;
  if (g >= groups) return;
  const int r0 = blockIdx.x * kRowsPerChunk;
  const int r1 = min(T, r0 + kRowsPerChunk);
  int cs = -1, cm = -1;
  float a_shift[8], a_scale[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) a_shift[e] = a_scale[e] = 0.f;
  auto flush = [&]() {
    float* base = dmod + ((static_cast<size_t>(cs) * 2 + cm) * 3) * hid + 8 * g;
    atomic_add8(base, a_shift);        // SHIFT slot
    atomic_add8(base + hid, a_scale);  // SCALE slot
  };
  for (int t = r0; t < r1; ++t) {
    int s, m;
    if (!token_ids(tok_sample, tok_mod, t, S, s, m, ctl)) continue;
    if (s != cs || m != cm) {
      if (cs >= 0) flush();
      cs = s;
      cm = m;
#pragma unroll
      for (int e = 0; e < 8; ++e) a_shift[e] = a_scale[e] = 0.f;
    }
    const float2 st = __ldg(stats + t);
    const size_t off = static_cast<size_t>(t) * groups + g;
    float f[8], d[8];
    unpack8(__ldg(x + off), f);
    unpack8(__ldg(dxm + off), d);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      a_shift[e] += d[e];
      a_scale[e] = fmaf(d[e], (f[e] - st.x) * st.y, a_scale[e]);
    }
  }
  if (cs >= 0) flush();
}

// ------------------------------------------------ modulation-map backward
constexpr int kDwRows = 16;      // rows of dW per thread
constexpr int kDwSamples = 8;    // samples staged per pass
constexpr int kDwThreads = 128;
constexpr int kDcThreads = 256;
constexpr int kDcSamples = 8;    // dot products per pass over W's row

// dW[r][n] = sum_s c[s][r] * dmod[s][n]. grid: (N4 / kDwThreads, C / kDwRows).
__global__ void __launch_bounds__(kDwThreads) params_dw_kernel(
    const float4* __restrict__ dmod4, const float* __restrict__ c, int S, int C, int N4,
    float4* __restrict__ dW4) {
  __shared__ float s_c[kDwSamples][kDwRows];
  const int n4 = blockIdx.x * kDwThreads + threadIdx.x;
  const int r0 = blockIdx.y * kDwRows;
  float4 acc[kDwRows];
#pragma unroll
  for (int r = 0; r < kDwRows; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < S; s0 += kDwSamples) {
    const int ns = min(kDwSamples, S - s0);
    __syncthreads();
    for (int i = threadIdx.x; i < kDwSamples * kDwRows; i += kDwThreads) {
      const int u = i / kDwRows, r = i % kDwRows;
      s_c[u][r] = (u < ns && r0 + r < C) ? c[static_cast<size_t>(s0 + u) * C + r0 + r] : 0.f;
    }
    __syncthreads();
    if (n4 < N4) {
      for (int u = 0; u < ns; ++u) {
        const float4 d = __ldg(dmod4 + static_cast<size_t>(s0 + u) * N4 + n4);
#pragma unroll
        for (int r = 0; r < kDwRows; ++r) {
          const float cv = s_c[u][r];
          acc[r].x = fmaf(cv, d.x, acc[r].x);
          acc[r].y = fmaf(cv, d.y, acc[r].y);
          acc[r].z = fmaf(cv, d.z, acc[r].z);
          acc[r].w = fmaf(cv, d.w, acc[r].w);
        }
      }
    }
  }
  if (n4 < N4) {
#pragma unroll
    for (int r = 0; r < kDwRows; ++r)
      if (r0 + r < C) dW4[static_cast<size_t>(r0 + r) * N4 + n4] = acc[r];
  }
}

// dc[s][r] = sum_n dmod[s][n] * W[r][n]. grid: C CTAs (one row of W each).
__global__ void __launch_bounds__(kDcThreads) params_dc_kernel(
    const float4* __restrict__ dmod4, const float4* __restrict__ W4, int S, int C, int N4,
    float* __restrict__ dc) {
  __shared__ float s_part[kDcThreads / 32][kDcSamples];
  const int r = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float4* wrow = W4 + static_cast<size_t>(r) * N4;
  for (int s0 = 0; s0 < S; s0 += kDcSamples) {
    const int ns = min(kDcSamples, S - s0);
    float acc[kDcSamples];
#pragma unroll
    for (int u = 0; u < kDcSamples; ++u) acc[u] = 0.f;
    for (int n4 = threadIdx.x; n4 < N4; n4 += kDcThreads) {
      const float4 wv = __ldg(wrow + n4);
#pragma unroll
      for (int u = 0; u < kDcSamples; ++u) {
        if (u < ns) {
          const float4 d = __ldg(dmod4 + static_cast<size_t>(s0 + u) * N4 + n4);
          acc[u] = fmaf(d.x, wv.x, fmaf(d.y, wv.y, fmaf(d.z, wv.z, fmaf(d.w, wv.w, acc[u]))));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kDcSamples; ++u) acc[u] = warp_sum(acc[u]);
    __syncthreads();  // the previous pass has read s_part
    if (lane == 0)
#pragma unroll
      for (int u = 0; u < kDcSamples; ++u) s_part[warp][u] = acc[u];
    __syncthreads();
    if (threadIdx.x < ns) {
      float v = 0.f;
#pragma unroll
      for (int wi = 0; wi < kDcThreads / 32; ++wi) v += s_part[wi][threadIdx.x];
      dc[static_cast<size_t>(s0 + threadIdx.x) * C + r] = v;
    }
  }
}

cudaError_t zero_slots(float* dmod, int32_t S, int32_t hid, int slot_mask, cudaStream_t st) {
  const long long n = static_cast<long long>(S) * 6 * hid;
  long long blocks = (n + 255) / 256;
  const long long cap = static_cast<long long>(sm_count()) * 4;
  if (blocks > cap) blocks = cap;
  zero_mod_slots_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(dmod, n, hid, slot_mask);
  return cudaGetLastError();
}

dim3 col_grid(int32_t T, int32_t hid) {
  const int groups = hid / 8;
  return dim3(static_cast<unsigned>((T + kRowsPerChunk - 1) / kRowsPerChunk),
              static_cast<unsigned>((groups + kColThreads - 1) / kColThreads));
}

}  // namespace

cudaError_t launch_gated_residual_bwd(const mf_bf16* dy, const mf_bf16* o, const float* mod,
                                      const int32_t* tok_sample, const uint8_t* tok_mod,
                                      int32_t T, int32_t S, int32_t hid, mf_bf16* d_o,
                                      float* dmod, const KernelCtl& ctl, cudaStream_t st) {
  cudaError_t e = zero_slots(dmod, S, hid, 1 << 2, st);
  if (e != cudaSuccess || T == 0) return e;
  gate_bwd_kernel<<<col_grid(T, hid), kColThreads, 0, st>>>(
      reinterpret_cast<const uint4*>(dy), reinterpret_cast<const uint4*>(o), mod, tok_sample,
      tok_mod, T, S, hid, reinterpret_cast<uint4*>(d_o), dmod, ctl);
  return cudaGetLastError();
}

cudaError_t launch_adaln_params_bwd(const float* dmod, const float* c, const float* W,
                                    int32_t S, int32_t C, int32_t hid, float* dc, float* dW,
                                    cudaStream_t st) {
  const int N4 = 6 * hid / 4;
  auto D4 = reinterpret_cast<const float4*>(dmod);
  if (dW != nullptr) {
    const dim3 grid(static_cast<unsigned>((N4 + kDwThreads - 1) / kDwThreads),
                    static_cast<unsigned>((C + kDwRows - 1) / kDwRows));
    params_dw_kernel<<<grid, kDwThreads, 0, st>>>(D4, c, S, C, N4, reinterpret_cast<float4*>(dW));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (dc != nullptr) {
    params_dc_kernel<<<C, kDcThreads, 0, st>>>(D4, reinterpret_cast<const float4*>(W), S, C, N4,
                                               dc);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

cudaError_t launch_adaln_modulate_bwd(const mf_bf16* dx_mod, const mf_bf16* x, const float* mod,
                                      const int32_t* tok_sample, const uint8_t* tok_mod,
                                      const mf_bf16* resid, int32_t T, int32_t S, int32_t hid,
                                      float eps, mf_bf16* dx, float* dmod, float* stats,
                                      const KernelCtl& ctl, cudaStream_t st) {
  cudaError_t e = zero_slots(dmod, S, hid, (1 << 0) | (1 << 1), st);
  if (e != cudaSuccess || T == 0) return e;
  long long blocks = (static_cast<long long>(T) + 7) / 8;
  const long long cap = static_cast<long long>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  ln_bwd_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      reinterpret_cast<const uint4*>(dx_mod), reinterpret_cast<const uint4*>(x),
      reinterpret_cast<const uint4*>(resid), mod, tok_sample, tok_mod, T, S, hid, eps,
      reinterpret_cast<uint4*>(dx), reinterpret_cast<float2*>(stats), ctl);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ln_bwd_cols_kernel<<<col_grid(T, hid), kColThreads, 0, st>>>(
      reinterpret_cast<const uint4*>(dx_mod), reinterpret_cast<const uint4*>(x),
      reinterpret_cast<const float2*>(stats), tok_sample, tok_mod, T, S, hid, dmod, ctl);
  return cudaGetLastError();
}

}  // namespace mf
