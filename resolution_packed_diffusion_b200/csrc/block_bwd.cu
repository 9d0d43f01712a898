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
  for (int t = r0; t < r1; ++t) {
    int s, m;
    if (!token_ids(tok_sample, tok_mod, t, S, s, m, ctl)) continue;
    if (s != cs || m != cm) {
      if (cs >= 0) atomic_add8(dmod + ((static_cast<size_t>(cs) * 2 + cm) * 3 + 2) * hid + 8 * g, acc);
      cs = s;
      cm = m;
      load8f(mod + ((static_cast<size_t>(s) * 2 + m) * 3 + 2) * hid + 8 * g, gate);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    }
    const size_t off = static_cast<size_t>(t) * groups + g;
    float fy[8], fo[8], out[8];
    unpack8(dy[off], fy);
    unpack8(__ldg(o + off), fo);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      acc[e] = fmaf(fy[e], fo[e], acc[e]);
      out[e] = gate[e] * fy[e];
    }
    d_o[off] = pack8(out);
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
