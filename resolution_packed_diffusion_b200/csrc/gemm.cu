// gemm.cu -- the modality-specific linear layer of the MMDiT block on sm_100a
// tensor cores: out[t] = x[t] W[m(t)]^T, m(t) the token's modality (0 image,
// 1 text), W stored [2][N][K].
//
// Source (page title, section): picx.dev "Mage-Flow" summary, Methodology >
// Native-Resolution MMDiT (an MMDiT with modality-specific normalization and
// joint self-attention: the image and the text stream keep their own weights).
//
// Design (one persistent CTA per SM, 8 warps). The output is cut into R-row x
// 256-column tiles; an R-row block of the pack whose tokens are all of one
// modality is one job per column tile; a block that holds both modalities (at
// an image / text boundary) is two jobs, each computed with its modality's
// weights and writing only its own rows.
//   warp 0      TMA producer: 128 x 64 slices of x and 64-wide K slices of W
//               (128-byte swizzle, no multicast) into a ring of stages.
//   warp 1      tcgen05 issuer: D (fp32, TMEM) += A B^T with N = 256, K = 16,
//               both operands K-major in shared memory; two TMEM accumulators
//               of 256 columns alternate between jobs so that a job's
//               epilogue overlaps the next job's MMAs.
//   warps 2..3  idle.
//   warps 4..7  epilogue: one output row per thread (its TMEM lane), 32 columns
//               at a time, rounded to bf16 and stored if the row exists and is
//               of the job's modality.
// Two forms:
//   single  R = 128, M = 128: each CTA loads 128 x 64 of x and 256 x 64 of W
//           per K step (48 KB, 4 stages).
//   pair    R = 256 over a cluster of two CTAs on two SMs (cta_group::2): the
//           leader issues M = 256 MMAs; each CTA loads its own 128 rows of x
//           and half of the weight tile (128 output columns), 32 KB per K step
//           (7 stages), and keeps its 128 rows of the accumulator in its own
//           TMEM. Per SM the same MMA work needs a third fewer operand bytes
//           from L2, the limit of the single form.
// Units (job, column tile) are walked in column blocks of up to 12 tiles, every
// row block inside a block: a block of weights stays in L2 while x streams past
// it once per block (see unit_coords). Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>
#include <vector>

#include "gemm_internal.h"
#include "mf_internal.h"
#include "mf_ptx.cuh"

namespace mf {

namespace {

constexpr int GM = 128;             // rows of x per CTA (MMA M of the single form)
constexpr int GN = 256;             // output columns per tile (MMA N)
constexpr int GK = 64;              // K per stage: one 128-byte swizzle atom
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;  // two accumulators of GN columns

template <bool PAIR>
struct GemmLayout {
  static constexpr int ROWS = PAIR ? 2 * GM : GM;   // rows of a job
  static constexpr int B_ROWS = PAIR ? GN / 2 : GN;  // weight rows this CTA loads
  static constexpr int STAGES = PAIR ? 7 : 4;
  static constexpr int A_BYTES = GM * GK * 2;
  static constexpr int B_BYTES = B_ROWS * GK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t kPeers = PAIR ? 2 : 1;  // CTAs whose epilogue warps arrive
  static constexpr int OFF_STAGES = 0;
  static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
  // With PAIR the leader's FULL barriers count both CTAs' bytes and its
  // ACC_EMPTY both CTAs' epilogue warps; EMPTY and ACC_FULL arrive in both CTAs
  // from the leader's multicast commits.
  static constexpr int B_FULL = 0;                      // [STAGES]
  static constexpr int B_EMPTY = B_FULL + STAGES;       // [STAGES]
  static constexpr int B_ACC_FULL = B_EMPTY + STAGES;   // [2]
  static constexpr int B_ACC_EMPTY = B_ACC_FULL + 2;    // [2], one arrival per epilogue warp
  static constexpr int B_DRAIN = B_ACC_EMPTY + 2;
  static constexpr int NUM_BARS = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem slot, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget of one CTA");
};

struct GemmArgs {
  GemmJobs jobs;
  int32_t T, K, N;
  int32_t nb;  // column tiles per block of the traversal (divides N / GN)
  int32_t act;  // 0: none, 1: GELU (tanh form)
  const uint8_t* tok_mod;
  mf_bf16* out;
  KernelCtl ctl;
};

// L2 cache policy for the weight slices: re-read by every row tile, they are
// kept in L2 (evict_last) while the output streams past it (streaming stores).
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 2D tiled TMA load with an L2 cache policy (no multicast).
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int32_t x, int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// The same into this CTA's shared memory, completing on the pair leader's
// mbarrier (a cluster address). No multicast.
__device__ __forceinline__ void tma_load_2d_pair_hint(void* dst, const CUtensorMap* map,
                                                      uint32_t leader_bar, int32_t x, int32_t y,
                                                      uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// Unit u of the traversal -> (job, column tile): column tiles in blocks of nb;
// inside a block every job (row tile) in turn, the block's column tiles of a
// job back to back. The ~148 units in flight then cover about 148 / nb row
// tiles and one block of weights, which stays in L2 while x streams once per
// block.
__device__ __forceinline__ void unit_coords(int u, int n_jobs, int nb, int& job_idx, int& nt) {
  const int per_block = n_jobs * nb;
  const int b = u / per_block;
  const int r = u - b * per_block;
  job_idx = r / nb;
  nt = b * nb + (r - job_idx * nb);
}

// GELU, tanh form: 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))).
__device__ __forceinline__ float gelu_tanh(float y) {
  const float u = 0.7978845608028654f * fmaf(0.044715f * y, y * y, y);
  return 0.5f * y * (1.f + tanhf(u));
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

template <bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    modality_linear_kernel(const __grid_constant__ CUtensorMap tmap_x,
                           const __grid_constant__ CUtensorMap tmap_w,
                           const __grid_constant__ GemmArgs args) {
  using L = GemmLayout<PAIR>;
  constexpr int kStages = L::STAGES;
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
      tmem_alloc_pair(tmem_slot, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, kTmemCols);
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
  const int nN = args.N / GN;
  const int nK = args.K / GK;
  const int units = args.jobs.n * nN;
  // With PAIR the pair is the scheduling unit; rank r holds rows r * 128 ..
  // r * 128 + 127 of every job and output columns r * 128 .. of every tile's B.
  const int rank = PAIR ? static_cast<int>(cluster_ctarank()) : 0;
  const int unit0 = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int n_units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (warp == 0) {
    // ============================================================ TMA producer
    if (lane == 0) {
      const uint64_t keep = policy_evict_last();
      uint32_t it = 0;
      bool ok = true;
      for (int u = unit0; u < units && ok; u += n_units) {
        int ji, nt;
        unit_coords(u, args.jobs.n, args.nb, ji, nt);
        const int job = args.jobs.job[ji];
        const int blk = job & 0x7fff, m = job >> 15;
        const int xr = blk * L::ROWS + rank * GM;
        const int wr = m * args.N + nt * GN + rank * L::B_ROWS;
        for (int kb = 0; kb < nK; ++kb, ++it) {
          const int st = it % kStages;
          if (!mbar_wait(&bars[L::B_EMPTY + st], ((it / kStages) & 1) ^ 1, args.ctl, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + L::OFF_STAGES + st * L::STAGE_BYTES;
          if constexpr (PAIR) {
            // both CTAs' halves complete on the leader's FULL barrier, which the
            // leader's producer arms for both (a copy that lands first only takes
            // the barrier's byte count below zero for a while)
            if (rank == 0) mbar_expect_tx(&bars[L::B_FULL + st], 2 * L::STAGE_BYTES);
            const uint32_t lb = cluster_addr(&bars[L::B_FULL + st], 0);
            tma_load_2d_pair(sa, &tmap_x, lb, kb * GK, xr);
            tma_load_2d_pair_hint(sa + L::A_BYTES, &tmap_w, lb, kb * GK, wr, keep);
          } else {
            mbar_expect_tx(&bars[L::B_FULL + st], L::STAGE_BYTES);
            tma_load_2d(sa, &tmap_x, &bars[L::B_FULL + st], kb * GK, xr);
            tma_load_2d_hint(sa + L::A_BYTES, &tmap_w, &bars[L::B_FULL + st], kb * GK, wr, keep);
          }
        }
      }
      // Every copy this thread started lands before the CTA can exit. With
      // PAIR all copies complete on the leader's barriers: the leader drains
      // them for both CTAs, and the closing cluster barrier keeps rank 1 alive
      // until then.
      if (rank == 0)
        for (int st = 0; st < kStages; ++st)
          if (it > static_cast<uint32_t>(st)) {
            const uint32_t last = it - 1 - ((it - 1 - st) % kStages);
            drain_wait(&bars[L::B_FULL + st], (last / kStages) & 1, args.ctl.wait_limit_ns);
          }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    // With PAIR only the leader issues; every commit that a CTA's producer or
    // epilogue waits on is multicast to both CTAs.
    if (lane == 0 && rank == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(L::ROWS, GN, 0, 0);
      const uint32_t base = smem_u32(smem + L::OFF_STAGES);
      const uint64_t desc0 = sdesc_sw128(base, 16, 1024);
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
        if (!mbar_wait(&bars[L::B_ACC_EMPTY + acc], ((ul >> 1) & 1) ^ 1, args.ctl, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * GN;
        for (int kb = 0; kb < nK; ++kb, ++it) {
          const int st = it % kStages;
          if (!mbar_wait(&bars[L::B_FULL + st], (it / kStages) & 1, args.ctl, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = desc0 + static_cast<uint64_t>((st * L::STAGE_BYTES) >> 4);
          const uint64_t b0 = desc0 + static_cast<uint64_t>((st * L::STAGE_BYTES + L::A_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < GK / 16; ++kk) {  // a 16-element K step is 32 bytes inside the atom
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
    const int row = wq * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    uint32_t ul = 0;
    for (int u = unit0; u < units; u += n_units, ++ul) {
      int ji, nt;
      unit_coords(u, args.jobs.n, args.nb, ji, nt);
      const int job = args.jobs.job[ji];
      const int blk = job & 0x7fff, m = job >> 15;
      const uint32_t acc = ul & 1;
      if (!warp_wait(&bars[L::B_ACC_FULL + acc], (ul >> 1) & 1, args.ctl, abort_flag)) break;
      tc_fence_after();
      const int t = blk * L::ROWS + rank * GM + row;
      const bool keep = t < args.T && (args.tok_mod == nullptr || __ldg(args.tok_mod + t) == m);
      uint4* orow = reinterpret_cast<uint4*>(args.out + static_cast<size_t>(t) * args.N + nt * GN);
#pragma unroll 1
      for (int cc = 0; cc < GN; cc += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + acc * GN + cc, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) asm volatile("" : "+r"(v[e]));
        if (args.act == 1) {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(gelu_tanh(__uint_as_float(v[e])));
        }
        if (keep) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
            o.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
            o.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
            o.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
            __stcs(orow + cc / 8 + q, o);
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
    if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
  } else {
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
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

// [rows][cols] bf16, box = 64 columns x box_rows rows, 128-byte swizzle; rows
// past the end read as zeros.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int sms() {
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

template <bool PAIR>
bool kernel_ready(int dev) {
  static bool attr_set[64] = {false};
  if (dev < 0 || dev >= 64) return false;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(modality_linear_kernel<PAIR>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmLayout<PAIR>::SMEM_BYTES) != cudaSuccess)
      return false;
    attr_set[dev] = true;
  }
  return true;
}

cudaLaunchConfig_t pair_config(int clusters, cudaLaunchAttribute* attr, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = GemmLayout<true>::SMEM_BYTES;
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
int max_clusters(int dev) {
  static int cached[64] = {0};
  if (dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    if (!kernel_ready<true>(dev)) return 0;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pair_config(1, attr, nullptr);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, modality_linear_kernel<true>, &cfg) != cudaSuccess ||
        n <= 0)
      return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

}  // namespace

int gemm_job_rows(bool pair) { return pair ? 2 * GM : GM; }

bool build_gemm_jobs(const int32_t* mods_per_sample_img, const int32_t* mods_per_sample_txt,
                     int32_t S, int32_t T, int32_t rows, GemmJobs* jobs) {
  if (rows != GM && rows != 2 * GM) return false;
  const int tiles = (T + rows - 1) / rows;
  if (tiles > kMaxGemmTiles) return false;
  std::vector<uint8_t> has(static_cast<size_t>(tiles), 0);  // bit m: modality m present
  int64_t row = 0;
  for (int32_t s = 0; s < S; ++s) {
    const int64_t runs[2] = {mods_per_sample_img[s], mods_per_sample_txt[s]};
    for (int m = 0; m < 2; ++m) {
      if (runs[m] > 0) {
        for (int64_t tl = row / rows; tl <= (row + runs[m] - 1) / rows; ++tl) has[tl] |= 1u << m;
        row += runs[m];
      }
    }
  }
  if (row != T) return false;
  int n = 0;
  for (int tl = 0; tl < tiles; ++tl)
    for (int m = 0; m < 2; ++m)
      if (has[tl] & (1u << m)) jobs->job[n++] = static_cast<uint16_t>(tl | (m << 15));
  jobs->n = n;
  return true;
}

namespace {

// w_sets: weight matrices stacked in W (2 for the per-modality form, 1 when
// tok_mod is NULL and every row uses W[0]).
cudaError_t launch_linear_impl(const mf_bf16* x, const mf_bf16* W, int w_sets,
                               const uint8_t* tok_mod, const GemmJobs& jobs, bool pair, int32_t T,
                               int32_t K, int32_t N, int32_t act, mf_bf16* out,
                               const KernelCtl& ctl, cudaStream_t st) {
  if (jobs.n == 0) return cudaSuccess;
  CUtensorMap mx, mw;
  const int b_rows = pair ? GemmLayout<true>::B_ROWS : GemmLayout<false>::B_ROWS;
  if (!make_map(&mx, x, T, K, GM) || !make_map(&mw, W, static_cast<int64_t>(w_sets) * N, K, b_rows))
    return cudaErrorInvalidValue;
  static thread_local GemmArgs a;
  a.jobs = jobs;
  a.T = T;
  a.K = K;
  a.N = N;
  a.tok_mod = tok_mod;
  a.out = out;
  a.act = act;
  // column-tile block: the largest divisor of N / GN that is at most 12
  const int nN = N / GN;
  a.nb = 1;
  for (int d = 1; d <= 12 && d <= nN; ++d)
    if (nN % d == 0) a.nb = d;
  a.ctl = ctl;
  int dev = 0;
  cudaGetDevice(&dev);
  const int units = jobs.n * nN;
  if (pair) {
    const int mc = max_clusters(dev);
    if (mc <= 0) return cudaErrorInvalidConfiguration;
    const int clusters = units < mc ? units : mc;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pair_config(clusters, attr, st);
    return cudaLaunchKernelEx(&cfg, modality_linear_kernel<true>, mx, mw, a);
  }
  if (!kernel_ready<false>(dev)) return cudaErrorInvalidConfiguration;
  const int grid = units < sms() ? units : sms();
  modality_linear_kernel<false><<<grid, kThreads, GemmLayout<false>::SMEM_BYTES, st>>>(mx, mw, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_modality_linear(const mf_bf16* x, const mf_bf16* W, const uint8_t* tok_mod,
                                   const GemmJobs& jobs, bool pair, int32_t T, int32_t K,
                                   int32_t N, int32_t act, mf_bf16* out, const KernelCtl& ctl,
                                   cudaStream_t st) {
  return launch_linear_impl(x, W, 2, tok_mod, jobs, pair, T, K, N, act, out, ctl, st);
}

cudaError_t launch_linear_plain(const mf_bf16* x, const mf_bf16* W, int32_t T, int32_t K,
                                int32_t N, bool pair, mf_bf16* out, const KernelCtl& ctl,
                                cudaStream_t st) {
  static thread_local GemmJobs jobs;
  const int rows = gemm_job_rows(pair);
  const int blocks = (T + rows - 1) / rows;
  if (blocks > kMaxGemmTiles) return cudaErrorInvalidValue;
  for (int b = 0; b < blocks; ++b) jobs.job[b] = static_cast<uint16_t>(b);
  jobs.n = blocks;
  return launch_linear_impl(x, W, 1, nullptr, jobs, pair, T, K, N, 0, out, ctl, st);
}

}  // namespace mf
