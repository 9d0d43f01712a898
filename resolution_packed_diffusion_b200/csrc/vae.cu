// vae.cu -- the Mage-VAE conv block's fused chains on sm_100a: GroupNorm + SiLU
// as one normalise-and-activate pass, and the 3x3 convolution as an implicit
// GEMM on tcgen05 tensor cores with the bias and the residual fused into its
// epilogue.
//
// Sources (page title, section): picx.dev "Mage-Flow" summary, Methodology >
// Mage-VAE, "Architecture" (a fully convolutional one-step diffusion decoder
// of stacked convolutional blocks, no global attention; 16x downsampled,
// 128-channel latents) and Methodology > Training Infrastructure (the stack's
// CUDA kernels fuse the normalization - activation - residual chains of the
// VAE's repeated blocks). The block's wiring is not on the pages; the library
// takes the diffusion conv nets' residual block:
//   y = x + conv3x3(SiLU(GN(h)); W2, c2),  h = conv3x3(SiLU(GN(x)); W1, c1).
// Layout NHWC bf16 (channels innermost); conv weights [Cout][3][3][Cin] bf16;
// GroupNorm affine parameters and conv biases fp32.
//
// Kernels:
//   gn_partial_kernel   per (pixel chunk, sample): each thread sums its
//                       8-channel vectors' values and squares about one of its
//                       own values and turns them into (count, mean, M2); the
//                       CTA merges those per group in a fixed order (Chan's
//                       pairwise update) and writes one partial per group.
//   gn_finalize_kernel  one CTA per (sample, group): merges the chunks'
//                       partials in a fixed tree -> (mean, rstd). Deterministic.
//   gn_silu_kernel      y = SiLU((x - mean) rstd gamma + beta), 16-byte vectors;
//                       a thread keeps one 8-channel vector over a run of pixels.
//   conv3x3_kernel<GN>  one persistent CTA per SM, 8 warps: output tiles of 128
//                       pixels (a BH x BW block of one image) x GN output
//                       channels (256, else 128, else 64: the widest that
//                       divides Cout); K runs over 9 taps x Cin / 64 channel blocks.
//                       warp 0 loads, per K step, the 128 input pixels the tap
//                       reads (a 4D TMA box {64 channels, BW, BH, 1} at
//                       (c, w0 + dx - 1, h0 + dy - 1, n): coordinates outside
//                       the image read as zeros, which is the zero padding) and
//                       the tap's GN x 64 weight slice, into a 4-stage ring;
//                       warp 1 issues M = 128, N = GN, K = 16 MMAs into one of
//                       two TMEM accumulators; warps 4..7 add the bias and the
//                       residual and store bf16 rows of valid pixels.
//                       With CTA pairs (cta_group::2) a cluster of two CTAs on
//                       two SMs computes two vertically adjacent pixel tiles
//                       (2 BH x BW) as M = 256 MMAs issued by the leader: each
//                       CTA loads its own tile's input boxes and half of each
//                       weight slice (GN / 2 rows), so each SM loads a quarter
//                       to a third fewer operand bytes per FLOP.
// Every wait is bounded; a CTA whose wait runs out records MF_ERR_TIMEOUT and
// winds down.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "mf_internal.h"
#include "mf_ptx.cuh"
#include "vae_internal.h"

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

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// ------------------------------------------------------------ GroupNorm
// (count, mean, M2) of a set of values; merge() is Chan et al.'s pairwise
// update, exact in real arithmetic and stable in floating point.
struct Moments {
  float n, mean, m2;
};
__device__ __forceinline__ Moments merge(const Moments& a, const Moments& b) {
  const float n = a.n + b.n;
  if (n == 0.f) return a;
  const float d = b.mean - a.mean;
  const float wb = b.n / n;
  return {n, fmaf(d, wb, a.mean), a.m2 + b.m2 + d * d * a.n * wb};
}

constexpr int kGnThreads = 256;

// grid (chunks, N); partial[(n * chunks + chunk) * G + g] = moments of group g
// over the chunk's pixels. VP = C / 8 vectors per pixel divides 256.
__global__ void __launch_bounds__(kGnThreads) gn_partial_kernel(
    const uint4* __restrict__ x, int HW, int C, int G, int chunk_px, float4* __restrict__ partial) {
  __shared__ Moments s_m[kGnThreads];
  const int VP = C >> 3;
  const int rows = kGnThreads / VP;  // pixels in flight per CTA step
  const int v = threadIdx.x % VP;    // this thread's 8-channel vector
  const int r = threadIdx.x / VP;
  const int n = blockIdx.y;
  const int p0 = blockIdx.x * chunk_px;
  const int p1 = min(HW, p0 + chunk_px);
  // this thread's pixels: sums of (value - K) and its square, K = its first
  // value (a sample of the data keeps the shifted sums well conditioned), turned
  // into (count, mean, M2) once at the end
  const uint4* xs = x + static_cast<size_t>(n) * HW * VP;
  float K = 0.f, s1 = 0.f, s2 = 0.f, cnt = 0.f;
  if (p0 + r < p1) K = __uint_as_float(__ldg(xs + static_cast<size_t>(p0 + r) * VP + v).x << 16);
#pragma unroll 4
  for (int p = p0 + r; p < p1; p += rows) {
    float f[8];
    unpack8(__ldg(xs + static_cast<size_t>(p) * VP + v), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float d = f[e] - K;
      s1 += d;
      s2 = fmaf(d, d, s2);
    }
    cnt += 8.f;
  }
  Moments m = {0.f, 0.f, 0.f};
  if (cnt > 0.f) {
    const float dm = s1 / cnt;
    m = Moments{cnt, K + dm, fmaxf(s2 - s1 * dm, 0.f)};
  }
  s_m[threadIdx.x] = m;
  __syncthreads();
  // per vector: merge the rows in order; then per group: its vectors in order
  if (threadIdx.x < VP) {
    Moments a = s_m[threadIdx.x];
    for (int rr = 1; rr < rows; ++rr) a = merge(a, s_m[rr * VP + threadIdx.x]);
    s_m[threadIdx.x] = a;
  }
  __syncthreads();
  const int vpg = VP / G;  // vectors per group
  for (int g = threadIdx.x; g < G; g += kGnThreads) {
    Moments a = s_m[g * vpg];
    for (int u = 1; u < vpg; ++u) a = merge(a, s_m[g * vpg + u]);
    partial[(static_cast<size_t>(n) * gridDim.x + blockIdx.x) * G + g] =
        make_float4(a.n, a.mean, a.m2, 0.f);
  }
}

// one CTA per (sample, group): each thread merges the chunks t, t + 256, ...
// in order, then the CTA merges the threads' moments pairwise in a fixed tree
// -> stats[n * G + g] = (mean, rstd). The same order every call.
__global__ void __launch_bounds__(kGnThreads) gn_finalize_kernel(const float4* __restrict__ partial,
                                                                 int G, int chunks, float eps,
                                                                 float2* __restrict__ stats) {
  __shared__ Moments s_m[kGnThreads];
  const int n = blockIdx.x / G, g = blockIdx.x - n * G;
  Moments a = {0.f, 0.f, 0.f};
  for (int c = threadIdx.x; c < chunks; c += kGnThreads) {
    const float4 p = __ldg(partial + (static_cast<size_t>(n) * chunks + c) * G + g);
    a = merge(a, Moments{p.x, p.y, p.z});
  }
  s_m[threadIdx.x] = a;
  __syncthreads();
  for (int half = kGnThreads / 2; half > 0; half >>= 1) {
    if (threadIdx.x < half) s_m[threadIdx.x] = merge(s_m[threadIdx.x], s_m[threadIdx.x + half]);
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const Moments m = s_m[0];
    const float var = m.n > 0.f ? m.m2 / m.n : 0.f;
    stats[blockIdx.x] = make_float2(m.mean, rsqrtf(var + eps));
  }
}

// y = SiLU((x - mean) * rstd * gamma + beta), one 8-channel vector per step
// grid: (pixel chunks, samples). A thread keeps one 8-channel vector v of the
// pixels and walks pixels p0 + r, p0 + r + rows, ... of its chunk, so its
// group's (mean, rstd) and its channels' gamma and beta are loaded once.
__global__ void __launch_bounds__(256) gn_silu_kernel(const uint4* __restrict__ x,
                                                      const float* __restrict__ gamma,
                                                      const float* __restrict__ beta,
                                                      const float2* __restrict__ stats, int HW,
                                                      int C, int G, int chunk_px,
                                                      uint4* __restrict__ y) {
  const int VP = C >> 3;          // a power of two <= 256, so it divides the block
  const int rows = blockDim.x / VP;
  const int v = threadIdx.x % VP, r = threadIdx.x / VP;
  const int n = blockIdx.y;
  const int c0 = 8 * v;
  const float2 st = __ldg(stats + n * G + c0 / (C / G));  // a vector never straddles groups
  float gm[8], bt[8];
  {
    const float4 g0 = __ldg(reinterpret_cast<const float4*>(gamma + c0));
    const float4 g1 = __ldg(reinterpret_cast<const float4*>(gamma + c0 + 4));
    const float4 b0 = __ldg(reinterpret_cast<const float4*>(beta + c0));
    const float4 b1 = __ldg(reinterpret_cast<const float4*>(beta + c0 + 4));
    gm[0] = g0.x; gm[1] = g0.y; gm[2] = g0.z; gm[3] = g0.w;
    gm[4] = g1.x; gm[5] = g1.y; gm[6] = g1.z; gm[7] = g1.w;
    bt[0] = b0.x; bt[1] = b0.y; bt[2] = b0.z; bt[3] = b0.w;
    bt[4] = b1.x; bt[5] = b1.y; bt[6] = b1.z; bt[7] = b1.w;
  }
  // the affine form of the normalisation: a = x * sc + sh
  float sc[8], sh[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    sc[e] = st.y * gm[e];
    sh[e] = fmaf(-st.x, sc[e], bt[e]);
  }
  const int p0 = blockIdx.x * chunk_px;
  const int p1 = min(HW, p0 + chunk_px);
  const size_t base = static_cast<size_t>(n) * HW * VP + v;
#pragma unroll 4
  for (int p = p0 + r; p < p1; p += rows) {
    const size_t i = base + static_cast<size_t>(p) * VP;
    float f[8];
    unpack8(__ldcs(x + i), f);
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float a0 = fmaf(f[2 * e], sc[2 * e], sh[2 * e]);
      float a1 = fmaf(f[2 * e + 1], sc[2 * e + 1], sh[2 * e + 1]);
      a0 = __fdividef(a0, 1.f + __expf(-a0));
      a1 = __fdividef(a1, 1.f + __expf(-a1));
      o[e] = pack_bf16x2(a0, a1);
    }
    __stcs(y + i, make_uint4(o[0], o[1], o[2], o[3]));
  }
}

// ------------------------------------------------------------ conv3x3
constexpr int CM = 128;            // output pixels per tile (MMA M)
constexpr int CK = 64;             // input channels per K step (one 128-byte atom)
constexpr int kConvThreads = 256;
constexpr int CA_BYTES = CM * CK * 2;  // A stage: 128 pixels x 64 channels

template <int GN, bool PAIR>
struct ConvLayout {
  static constexpr int B_ROWS = PAIR ? GN / 2 : GN;  // weight rows this CTA loads
  static constexpr int B_BYTES = B_ROWS * CK * 2;
  static constexpr int STAGE = CA_BYTES + B_BYTES;
  static constexpr int STAGES = (200 * 1024 / STAGE) < 8 ? (200 * 1024 / STAGE) : 8;
  static constexpr uint32_t kPeers = PAIR ? 2 : 1;  // CTAs whose epilogue warps arrive
  static constexpr int OFF_BAR = STAGES * STAGE;
  // With PAIR the leader's FULL barriers count both CTAs' bytes and its
  // ACC_EMPTY both CTAs' epilogue warps; EMPTY and ACC_FULL arrive in both CTAs
  // from the leader's multicast commits.
  static constexpr int B_FULL = 0;                      // [stages]
  static constexpr int B_EMPTY = B_FULL + STAGES;       // [stages]
  static constexpr int B_ACC_FULL = B_EMPTY + STAGES;   // [2]
  static constexpr int B_ACC_EMPTY = B_ACC_FULL + 2;    // [2], one arrival per epilogue warp
  static constexpr int B_DRAIN = B_ACC_EMPTY + 2;
  static constexpr int NUM_BARS = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget of one CTA");
};

struct ConvArgs {
  int32_t N, H, W, Cin, Cout;
  int32_t BH, BW;          // pixel tile: BH rows x BW columns of one image (BH * BW = 128)
  int32_t UH;              // rows of a unit's pixel block: BH, or 2 BH with CTA pairs
  int32_t tiles_h, tiles_w;  // unit blocks down and across an image
  const float* bias;       // [Cout] or NULL
  const mf_bf16* residual; // [N][H][W][Cout] or NULL
  mf_bf16* y;              // [N][H][W][Cout]
  KernelCtl ctl;
};

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c, int32_t w, int32_t h, int32_t n) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c), "r"(w), "r"(h), "r"(n)
      : "memory");
}

// The same into this CTA's shared memory, completing on the pair leader's
// mbarrier (a cluster address). No multicast.
__device__ __forceinline__ void tma_load_4d_pair(void* dst, const CUtensorMap* map,
                                                 uint32_t leader_bar, int32_t c, int32_t w,
                                                 int32_t h, int32_t n) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(c), "r"(w), "r"(h), "r"(n)
      : "memory");
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const KernelCtl& ctl,
                                          volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, ctl, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) return;
  }
}

// unit u -> (image n, tile row h0, tile column w0, output-channel tile nt):
// the output-channel tiles of one pixel tile are consecutive, so they share
// its input boxes in L2
__device__ __forceinline__ void conv_unit(const ConvArgs& a, int nN, int u, int& n, int& h0,
                                          int& w0, int& nt) {
  nt = u % nN;
  int t = u / nN;
  const int tw = t % a.tiles_w;
  t /= a.tiles_w;
  const int th = t % a.tiles_h;
  n = t / a.tiles_h;
  h0 = th * a.UH;
  w0 = tw * a.BW;
}

template <int GN, bool PAIR>
__global__ void __launch_bounds__(kConvThreads, 1)
    conv3x3_kernel(const __grid_constant__ CUtensorMap tmap_x,
                   const __grid_constant__ CUtensorMap tmap_w,
                   const __grid_constant__ ConvArgs args) {
  using L = ConvLayout<GN, PAIR>;
  constexpr int kConvStages = L::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NUM_BARS; ++i)
      mbar_init(&bars[i], (i == L::B_ACC_EMPTY || i == L::B_ACC_EMPTY + 1) ? 4u * L::kPeers : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmap_x);
    tma_prefetch_map(&tmap_w);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      // both CTAs' warp 1, the same slot offset: the pair's TMEM at one address
      tmem_alloc_pair(tmem_slot, 2 * GN);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, 2 * GN);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  // Both CTAs' barriers are initialised before either CTA's arrivals, commits
  // or copies can reach the other's.
  if constexpr (PAIR) cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nN = args.Cout / GN;
  const int units = args.N * args.tiles_h * args.tiles_w * nN;
  const int ncb = args.Cin / CK;
  const int nk = 9 * ncb;  // K steps per tile: taps x channel blocks
  // With PAIR the pair is the scheduling unit: rank r computes the pixel tile
  // r * BH rows below the unit's origin and loads weight rows r * GN / 2 ..
  const int rank = PAIR ? static_cast<int>(cluster_ctarank()) : 0;
  const int unit0 = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int n_units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (warp == 0) {
    // ============================================================ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int u = unit0; u < units && ok; u += n_units) {
        int n, h0, w0, nt;
        conv_unit(args, nN, u, n, h0, w0, nt);
        h0 += rank * args.BH;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int st = it % kConvStages;
          if (!mbar_wait(&bars[L::B_EMPTY + st], ((it / kConvStages) & 1) ^ 1, args.ctl,
                         abort_flag)) {
            ok = false;
            break;
          }
          const int tap = kb / ncb, cb = kb - tap * ncb;
          const int dy = tap / 3, dx = tap - dy * 3;
          uint8_t* sa = smem + st * L::STAGE;
          // channel coordinate cb * 64: a multiple of 64 elements (128 bytes)
          const int wrow = nt * GN + rank * L::B_ROWS;
          if constexpr (PAIR) {
            // both CTAs' copies complete on the leader's FULL barrier, which the
            // leader's producer arms for both (a copy that lands first only
            // takes the barrier's byte count below zero for a while)
            if (rank == 0) mbar_expect_tx(&bars[L::B_FULL + st], 2 * L::STAGE);
            const uint32_t lb = cluster_addr(&bars[L::B_FULL + st], 0);
            tma_load_4d_pair(sa, &tmap_x, lb, cb * CK, w0 + dx - 1, h0 + dy - 1, n);
            tma_load_2d_pair(sa + CA_BYTES, &tmap_w, lb, tap * args.Cin + cb * CK, wrow);
          } else {
            mbar_expect_tx(&bars[L::B_FULL + st], L::STAGE);
            tma_load_4d(sa, &tmap_x, &bars[L::B_FULL + st], cb * CK, w0 + dx - 1, h0 + dy - 1, n);
            tma_load_2d(sa + CA_BYTES, &tmap_w, &bars[L::B_FULL + st], tap * args.Cin + cb * CK,
                        wrow);
          }
        }
      }
      // Every copy this thread started lands before the CTA can exit. With
      // PAIR all copies complete on the leader's barriers: the leader drains
      // them for both CTAs, and the closing cluster barrier keeps rank 1 alive
      // until then.
      if (rank == 0)
        for (int st = 0; st < kConvStages; ++st)
          if (it > static_cast<uint32_t>(st)) {
            const uint32_t last = it - 1 - ((it - 1 - st) % kConvStages);
            drain_wait(&bars[L::B_FULL + st], (last / kConvStages) & 1, args.ctl.wait_limit_ns);
          }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    // With PAIR only the leader issues; every commit that a CTA's producer or
    // epilogue waits on is multicast to both CTAs.
    if (lane == 0 && rank == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(PAIR ? 2 * CM : CM, GN, 0, 0);
      const uint64_t desc0 = sdesc_sw128(smem_u32(smem), 16, 1024);
      auto commit = [&](int b) {
        if constexpr (PAIR)
          umma_commit_pair(&bars[b], 3);
        else
          umma_commit(&bars[b]);
      };
      uint32_t it = 0, ul = 0;
      bool ok = true;
      for (int u = unit0; u < units && ok; u += n_units, ++ul) {
        const uint32_t acc = ul & 1;
        if (!mbar_wait(&bars[L::B_ACC_EMPTY + acc], ((ul >> 1) & 1) ^ 1, args.ctl, abort_flag))
          break;
        tc_fence_after();
        const uint32_t d = tmem + acc * GN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int st = it % kConvStages;
          if (!mbar_wait(&bars[L::B_FULL + st], (it / kConvStages) & 1, args.ctl, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = desc0 + static_cast<uint64_t>((st * L::STAGE) >> 4);
          const uint64_t b0 = desc0 + static_cast<uint64_t>((st * L::STAGE + CA_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < CK / 16; ++kk) {  // a 16-element K step is 32 bytes in the atom
            if constexpr (PAIR)
              umma_ss_pair(d, a0 + kk * 2, b0 + kk * 2, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
            else
              umma_ss(d, a0 + kk * 2, b0 + kk * 2, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          commit(L::B_EMPTY + st);
        }
        if (!ok) break;
        commit(L::B_ACC_FULL + acc);
      }
      // every MMA this thread issued completes before TMEM is released
      if constexpr (PAIR)
        umma_commit_pair(&bars[L::B_DRAIN], 1);  // the leader's own barrier
      else
        umma_commit(&bars[L::B_DRAIN]);
      drain_wait(&bars[L::B_DRAIN], 0, args.ctl.wait_limit_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ============================================================ epilogue
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // pixel of the tile: (row / BW, row % BW)
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const int Cout = args.Cout;
    uint32_t ul = 0;
    for (int u = unit0; u < units; u += n_units, ++ul) {
      int n, h0, w0, nt;
      conv_unit(args, nN, u, n, h0, w0, nt);
      const int h = h0 + rank * args.BH + row / args.BW, w = w0 + row % args.BW;
      const bool valid = h < args.H && w < args.W;
      const size_t pix = (static_cast<size_t>(n) * args.H + (valid ? h : 0)) * args.W +
                         (valid ? w : 0);
      const uint32_t acc = ul & 1;
      if (!warp_wait(&bars[L::B_ACC_FULL + acc], (ul >> 1) & 1, args.ctl, abort_flag)) break;
      tc_fence_after();
      const int c_base = nt * GN;
#pragma unroll 1
      for (int cc = 0; cc < GN; cc += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + acc * GN + cc, v);
        tmem_ld_wait();
        if (valid) {
          const size_t off = pix * Cout + c_base + cc;  // 32 channels: four 16-byte vectors
          float r[32];
          if (args.residual != nullptr) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float f[8];
              unpack8(__ldg(reinterpret_cast<const uint4*>(args.residual + off) + q), f);
#pragma unroll
              for (int e = 0; e < 8; ++e) r[8 * q + e] = f[e];
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = 0.f;
          }
          if (args.bias != nullptr) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 b = __ldg(reinterpret_cast<const float4*>(args.bias + c_base + cc) + q);
              r[4 * q] += b.x;
              r[4 * q + 1] += b.y;
              r[4 * q + 2] += b.z;
              r[4 * q + 3] += b.w;
            }
          }
          uint4* out = reinterpret_cast<uint4*>(args.y + off);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]) + r[8 * q + 0],
                              __uint_as_float(v[8 * q + 1]) + r[8 * q + 1]);
            o.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]) + r[8 * q + 2],
                              __uint_as_float(v[8 * q + 3]) + r[8 * q + 3]);
            o.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]) + r[8 * q + 4],
                              __uint_as_float(v[8 * q + 5]) + r[8 * q + 5]);
            o.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]) + r[8 * q + 6],
                              __uint_as_float(v[8 * q + 7]) + r[8 * q + 7]);
            out[q] = o;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR)
          mbar_arrive_cluster(cluster_addr(&bars[L::B_ACC_EMPTY + acc], 0));
        else
          mbar_arrive(&bars[L::B_ACC_EMPTY + acc]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if constexpr (PAIR) {
    // The leader has drained its MMAs (which write rank 1's TMEM) and the
    // copies that complete on its barriers; neither CTA frees TMEM or leaves
    // before both are here.
    cluster_sync();
    if (warp == 1) tmem_dealloc_pair(tmem, 2 * GN);
  } else {
    if (warp == 1) tmem_dealloc(tmem, 2 * GN);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// NHWC input as a 4D tensor {C, W, H, N}; box {64 channels, BW, BH, 1}; 128-byte
// swizzle (a box lands as BH * BW rows of 128 bytes: the K-major A operand);
// coordinates outside the tensor read as zeros.
bool make_input_map(CUtensorMap* map, const void* x, int N, int H, int W, int C, int BH, int BW) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(W),
                              static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(N)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(C) * 2,
                                 static_cast<cuuint64_t>(W) * C * 2,
                                 static_cast<cuuint64_t>(H) * W * C * 2};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(CK), static_cast<cuuint32_t>(BW),
                             static_cast<cuuint32_t>(BH), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(x), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// weights [Cout][9 * Cin] (tap-major K); box {64, rows}
bool make_weight_map(CUtensorMap* map, const void* Wt, int Cout, int Cin, int rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(9) * Cin, static_cast<cuuint64_t>(Cout)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(9) * Cin * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(CK), static_cast<cuuint32_t>(rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(Wt), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <int GN, bool PAIR>
bool conv_ready(int dev) {
  static bool attr_set[64] = {false};
  if (dev < 0 || dev >= 64) return false;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(conv3x3_kernel<GN, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ConvLayout<GN, PAIR>::SMEM_BYTES) != cudaSuccess)
      return false;
    attr_set[dev] = true;
  }
  return true;
}

template <int GN>
cudaLaunchConfig_t conv_pair_config(int clusters, cudaLaunchAttribute* attr, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kConvThreads);
  cfg.dynamicSmemBytes = ConvLayout<GN, true>::SMEM_BYTES;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// Clusters of two that can be resident at once (0 if the pair form cannot run).
template <int GN>
int conv_max_clusters(int dev) {
  static int cached[64] = {0};
  if (dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    if (!conv_ready<GN, true>(dev)) return 0;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = conv_pair_config<GN>(1, attr, nullptr);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, conv3x3_kernel<GN, true>, &cfg) != cudaSuccess || n <= 0)
      return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

template <int GN>
cudaError_t launch_conv_t(const CUtensorMap& mx, const CUtensorMap& mw, const ConvArgs& a,
                          long long units, bool pair, cudaStream_t st) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (pair) {
    const int mc = conv_max_clusters<GN>(dev);
    if (mc <= 0) return cudaErrorInvalidConfiguration;
    const int clusters = units < mc ? static_cast<int>(units) : mc;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = conv_pair_config<GN>(clusters, attr, st);
    return cudaLaunchKernelEx(&cfg, conv3x3_kernel<GN, true>, mx, mw, a);
  }
  if (!conv_ready<GN, false>(dev)) return cudaErrorInvalidConfiguration;
  const int grid = units < sm_count() ? static_cast<int>(units) : sm_count();
  conv3x3_kernel<GN, false>
      <<<grid, kConvThreads, ConvLayout<GN, false>::SMEM_BYTES, st>>>(mx, mw, a);
  return cudaGetLastError();
}

}  // namespace

int gn_chunks(int32_t N, int32_t H, int32_t W) {
  // about four CTAs per SM over the whole tensor, at least 64 pixels a chunk
  const long long HW = static_cast<long long>(H) * W;
  long long c = (4LL * sm_count() + N - 1) / N;
  const long long max_c = (HW + 63) / 64;
  if (c > max_c) c = max_c;
  return static_cast<int>(c < 1 ? 1 : c);
}

size_t gn_workspace_bytes(int32_t N, int32_t H, int32_t W, int32_t G) {
  const size_t partial = static_cast<size_t>(N) * gn_chunks(N, H, W) * G * sizeof(float4);
  const size_t stats = static_cast<size_t>(N) * G * sizeof(float2);
  return ((partial + 255) / 256) * 256 + ((stats + 255) / 256) * 256;
}

cudaError_t launch_group_norm_silu(const mf_bf16* x, const float* gamma, const float* beta,
                                   int32_t N, int32_t H, int32_t W, int32_t C, int32_t G,
                                   float eps, mf_bf16* y, void* workspace, cudaStream_t st) {
  const int chunks = gn_chunks(N, H, W);
  const int HW = H * W;
  const int chunk_px = (HW + chunks - 1) / chunks;
  float4* partial = static_cast<float4*>(workspace);
  const size_t pbytes = static_cast<size_t>(N) * chunks * G * sizeof(float4);
  float2* stats = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) +
                                            ((pbytes + 255) / 256) * 256);
  gn_partial_kernel<<<dim3(chunks, N), kGnThreads, 0, st>>>(reinterpret_cast<const uint4*>(x), HW,
                                                            C, G, chunk_px, partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  gn_finalize_kernel<<<N * G, kGnThreads, 0, st>>>(partial, G, chunks, eps, stats);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // about eight 256-thread CTAs per SM over the whole tensor, each a run of pixels
  const int rows = 256 / (C / 8);
  long long nchunk = (8LL * sm_count() + N - 1) / N;
  const long long max_chunk = (HW + rows - 1) / rows;
  if (nchunk > max_chunk) nchunk = max_chunk;
  if (nchunk < 1) nchunk = 1;
  const int chunk_px2 = static_cast<int>((HW + nchunk - 1) / nchunk);
  gn_silu_kernel<<<dim3(static_cast<unsigned>(nchunk), N), 256, 0, st>>>(
      reinterpret_cast<const uint4*>(x), gamma, beta, stats, HW, C, G, chunk_px2,
      reinterpret_cast<uint4*>(y));
  return cudaGetLastError();
}

void conv_pixel_tile(int32_t H, int32_t W, int32_t* BH, int32_t* BW) {
  // the 128-pixel block (BH x BW, BW a power of two from 8 to 128) that
  // covers the image with the fewest computed pixels; wider on ties
  long long best = -1;
  for (int bw = 128; bw >= 8; bw /= 2) {
    const int bh = 128 / bw;
    const long long cost = static_cast<long long>((H + bh - 1) / bh) * bh * ((W + bw - 1) / bw) * bw;
    if (best < 0 || cost < best) {
      best = cost;
      *BH = bh;
      *BW = bw;
    }
  }
}

cudaError_t launch_conv3x3(const mf_bf16* x, const mf_bf16* Wt, const float* bias,
                           const mf_bf16* residual, int32_t N, int32_t H, int32_t W, int32_t Cin,
                           int32_t Cout, mf_bf16* y, bool pair, const KernelCtl& ctl,
                           cudaStream_t st) {
  static thread_local ConvArgs a;
  a.N = N;
  a.H = H;
  a.W = W;
  a.Cin = Cin;
  a.Cout = Cout;
  conv_pixel_tile(H, W, &a.BH, &a.BW);
  a.UH = pair ? 2 * a.BH : a.BH;
  a.tiles_h = (H + a.UH - 1) / a.UH;
  a.tiles_w = (W + a.BW - 1) / a.BW;
  a.bias = bias;
  a.residual = residual;
  a.y = y;
  a.ctl = ctl;
  const int gn = (Cout % 256 == 0) ? 256 : (Cout % 128 == 0 ? 128 : 64);
  CUtensorMap mx, mw;
  if (!make_input_map(&mx, x, N, H, W, Cin, a.BH, a.BW) ||
      !make_weight_map(&mw, Wt, Cout, Cin, pair ? gn / 2 : gn))
    return cudaErrorInvalidValue;
  const long long units = static_cast<long long>(N) * a.tiles_h * a.tiles_w * (Cout / gn);
  if (gn == 256) return launch_conv_t<256>(mx, mw, a, units, pair, st);
  if (gn == 128) return launch_conv_t<128>(mx, mw, a, units, pair, st);
  return launch_conv_t<64>(mx, mw, a, units, pair, st);
}

}  // namespace mf
