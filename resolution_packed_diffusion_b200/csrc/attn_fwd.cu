// attn_fwd.cu -- block-diagonal variable-length attention on sm_100a tensor
// cores (tcgen05 + TMEM, operands staged by TMA), with an optional fused gated
// residual epilogue.
//
// What it computes (picx.dev "Mage-Flow" summary, Methodology > Native-
// Resolution MMDiT: samples of a pack attend only inside their own token range,
// delimited by per-sample cumulative offsets; joint attention over the image and
// text tokens of a sample; Training Infrastructure: gating fused with the
// block): for every sample s and head h, O = softmax(Q K^T * scale) V over the
// sample's own keys; optionally y = x + gate[s, modality] * O.
//
// Design (one persistent CTA per SM, 6 warps):
//   warp 0      TMA producer: Q tile (128 rows) per work item, then K and V
//               tiles (128 rows) of the item's own sample only, in separate
//               rings (K slots free once S = Q K^T is done, V slots once PV is).
//   warp 1      tcgen05 issuer: S = Q K^T into one of two TMEM S buffers, then
//               O += P V with P read from TMEM (the A operand) and V from shared
//               memory (MN-major). Allocates / frees the 512 TMEM columns.
//   warps 2..5  softmax + epilogue, one thread per query row (TMEM lane): read S
//               from TMEM, online softmax in the exp2 domain with a lazy
//               rescale (O is rescaled only when the running max grows by more
//               than 2^8), write P as packed bf16 to TMEM, then O / l and the
//               epilogue from TMEM.
// Work items are (sample, head, 128-row query tile), ordered longest sample
// first and, inside a sample, query tiles of one head next to each other so
// that concurrently running CTAs stream the same K/V tiles through L2. Key tiles
// start at the sample's first token and never leave the sample: tiles of other
// samples are never visited; only the last key tile of a sample can be partial
// and only it is masked.
//
// Every wait is bounded (mbar_wait); on expiry the CTA records MF_ERR_TIMEOUT,
// lets its in-flight copies and MMAs finish, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "mf_internal.h"
#include "mf_ptx.cuh"

namespace mf {

namespace {

constexpr int BM = 128;              // query rows per tile (MMA M)
constexpr int BN = 128;              // key rows per tile (MMA N of QK^T, K of PV)
constexpr int NUM_THREADS = 192;     // 6 warps
constexpr uint32_t TMEM_COLS = 512;  // S0 | S1 | O | P0 | P1
constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O = 256, TM_P0 = 384, TM_P1 = 448;
constexpr int BOX_BYTES = 128 * 128;  // one TMA box: 128 rows x 64 bf16 (128 B), swizzled
constexpr int NK = 2;                 // K tile ring stages (freed after S = Q K^T)
constexpr int NV = 3;                 // V tile ring stages (freed after O += P V)
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: rescale O only past 2^8 growth

template <int D>
struct Layout {
  static constexpr int kBoxes = D / 64;  // 64-column boxes per 128-row tile
  static constexpr int TILE_BYTES = BM * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE_BYTES;
  static constexpr int OFF_V = OFF_K + NK * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + NV * TILE_BYTES;
  // barriers (arrival count 1 unless arrivals() says 4)
  static constexpr int B_Q_FULL = 0, B_Q_EMPTY = 1;
  static constexpr int B_K_FULL = 2;                 // NK
  static constexpr int B_K_EMPTY = B_K_FULL + NK;    // NK
  static constexpr int B_V_FULL = B_K_EMPTY + NK;    // NV
  static constexpr int B_V_EMPTY = B_V_FULL + NV;    // NV
  static constexpr int B_S_FULL = B_V_EMPTY + NV;    // 2
  static constexpr int B_S_FREE = B_S_FULL + 2;      // 2, one arrival per softmax warp
  static constexpr int B_P_FULL = B_S_FREE + 2;      // 2, one arrival per softmax warp
  static constexpr int B_PV_DONE = B_P_FULL + 2;     // 2
  static constexpr int B_O_FULL = B_PV_DONE + 2;
  static constexpr int B_O_EMPTY = B_O_FULL + 1;     // one arrival per softmax warp
  static constexpr int B_DRAIN = B_O_EMPTY + 1;
  static constexpr int NUM_BARS = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem slot, abort, bad flag
  static constexpr int OFF_CU = OFF_MISC + 16;
  static constexpr int OFF_ORDER = OFF_CU + (MF_MAX_SAMPLES + 1) * 4;
  static constexpr int OFF_ISTART = OFF_ORDER + MF_MAX_SAMPLES * 4;
  static constexpr int END = OFF_ISTART + (MF_MAX_SAMPLES + 1) * 4;
  // + alignment slack; at least 120 KB so that two CTAs never share an SM (each
  // holds all 512 TMEM columns, a second CTA would block in tcgen05.alloc)
  static constexpr int SMEM_BYTES = (END + 1024) > 120 * 1024 ? (END + 1024) : 120 * 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget of one CTA");

  __device__ static uint32_t arrivals(int i) {
    return (i == B_S_FREE || i == B_S_FREE + 1 || i == B_P_FULL || i == B_P_FULL + 1 ||
            i == B_O_EMPTY)
               ? 4u
               : 1u;
  }
};

struct AttnArgs {
  const int32_t* cu_seqlens;
  int32_t S, T, H;
  float scale_log2;  // softmax_scale * log2(e)
  AttnEpilogue ep;
  KernelCtl ctl;
};

struct WorkItem {
  int32_t s, qt, h, row0, kv0, n, nkv;
};

__device__ __forceinline__ WorkItem decode_item(int w, int S, int H, const int32_t* s_cu,
                                                const int32_t* s_order, const int32_t* s_istart) {
  int lo = 0, hi = S - 1;  // largest r with istart[r] <= w
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_istart[mid] <= w) lo = mid; else hi = mid - 1;
  }
  WorkItem it;
  it.s = s_order[lo];
  const int local = w - s_istart[lo];
  it.kv0 = s_cu[it.s];
  it.n = s_cu[it.s + 1] - it.kv0;
  const int nq = (it.n + BM - 1) / BM;
  it.h = local / nq;
  it.qt = local - it.h * nq;
  it.row0 = it.kv0 + it.qt * BM;
  it.nkv = (it.n + BN - 1) / BN;
  return it;
}

// Wait with every lane of a warp and agree on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const KernelCtl& ctl,
                                          volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, ctl, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait used while winding down: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) return;
  }
}

template <int D, bool GATED>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    varlen_attn_kernel(const __grid_constant__ CUtensorMap tmap_q,
                       const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v, const AttnArgs args) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte-swizzled TMA / UMMA tiles
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  volatile int* bad_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 8);
  int32_t* s_cu = reinterpret_cast<int32_t*>(smem + L::OFF_CU);
  int32_t* s_order = reinterpret_cast<int32_t*>(smem + L::OFF_ORDER);
  int32_t* s_istart = reinterpret_cast<int32_t*>(smem + L::OFF_ISTART);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = args.S, H = args.H;

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NUM_BARS; ++i) mbar_init(&bars[i], L::arrivals(i));
    *abort_flag = 0;
    *bad_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i <= S; i += NUM_THREADS) s_cu[i] = __ldg(args.cu_seqlens + i);
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmap_q);
    tma_prefetch_map(&tmap_k);
    tma_prefetch_map(&tmap_v);
  }
  __syncthreads();
  // validate the device offsets against the host's view of the pack
  for (int i = threadIdx.x; i < S; i += NUM_THREADS)
    if (s_cu[i + 1] < s_cu[i]) *bad_flag = 1;
  if (threadIdx.x == 0 && (s_cu[0] != 0 || s_cu[S] != args.T)) *bad_flag = 1;
  // longest-first order of the samples (rank sort; ties keep pack order)
  for (int i = threadIdx.x; i < S; i += NUM_THREADS) {
    const int ni = s_cu[i + 1] - s_cu[i];
    int rank = 0;
    for (int u = 0; u < S; ++u) {
      const int nu = s_cu[u + 1] - s_cu[u];
      rank += (nu > ni) || (nu == ni && u < i);
    }
    s_order[rank] = i;
  }
  __syncwarp();
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int r = 0; r < S; ++r) {
      s_istart[r] = acc;
      const int n = s_cu[s_order[r] + 1] - s_cu[s_order[r]];
      acc += ((n + BM - 1) / BM) * H;
    }
    s_istart[S] = acc;
    if (*bad_flag) atomicCAS(args.ctl.err, 0, static_cast<int>(MF_ERR_INVALID));
  }
  __syncthreads();
  const uint32_t tmem = *tmem_slot;
  const int total_items = *bad_flag ? 0 : s_istart[S];

  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;

  if (warp == 0) {
    // ============================================================ TMA producer
    // Order of loads: Q, K_0, then (K_{j+1}, V_j) -- the MMA warp consumes
    // S_j = Q K_j^T before O += P_{j-1} V_{j-1}, so K runs one tile ahead of V.
    if (lane == 0) {
      uint32_t kc = 0, vc = 0;  // K / V tiles issued so far (global over items)
      int n_item = 0;
      bool ok = true;
      auto load_k = [&](const WorkItem& wi, int j) -> bool {
        const int st = kc % NK;
        if (!mbar_wait(&bars[L::B_K_EMPTY + st], ((kc / NK) & 1) ^ 1, args.ctl, abort_flag)) return false;
        mbar_expect_tx(&bars[L::B_K_FULL + st], L::TILE_BYTES);
#pragma unroll
        for (int b = 0; b < L::kBoxes; ++b)
          tma_load_2d(sK + st * L::TILE_BYTES + b * BOX_BYTES, &tmap_k, &bars[L::B_K_FULL + st],
                      wi.h * D + 64 * b, wi.kv0 + j * BN);
        ++kc;
        return true;
      };
      auto load_v = [&](const WorkItem& wi, int j) -> bool {
        const int st = vc % NV;
        if (!mbar_wait(&bars[L::B_V_EMPTY + st], ((vc / NV) & 1) ^ 1, args.ctl, abort_flag)) return false;
        mbar_expect_tx(&bars[L::B_V_FULL + st], L::TILE_BYTES);
#pragma unroll
        for (int b = 0; b < L::kBoxes; ++b)
          tma_load_2d(sV + st * L::TILE_BYTES + b * BOX_BYTES, &tmap_v, &bars[L::B_V_FULL + st],
                      wi.h * D + 64 * b, wi.kv0 + j * BN);
        ++vc;
        return true;
      };
      for (int w = blockIdx.x; w < total_items && ok; w += gridDim.x, ++n_item) {
        const WorkItem wi = decode_item(w, S, H, s_cu, s_order, s_istart);
        if (!mbar_wait(&bars[L::B_Q_EMPTY], (n_item & 1) ^ 1, args.ctl, abort_flag)) break;
        mbar_expect_tx(&bars[L::B_Q_FULL], L::TILE_BYTES);
#pragma unroll
        for (int b = 0; b < L::kBoxes; ++b)
          tma_load_2d(sQ + b * BOX_BYTES, &tmap_q, &bars[L::B_Q_FULL], wi.h * D + 64 * b, wi.row0);
        if (!load_k(wi, 0)) break;
        for (int j = 0; j < wi.nkv; ++j) {
          if (j + 1 < wi.nkv && !load_k(wi, j + 1)) { ok = false; break; }
          if (!load_v(wi, j)) { ok = false; break; }
        }
      }
      // Let every copy this thread started land before the CTA can exit.
      const uint64_t lim = args.ctl.wait_limit_ns;
      if (n_item > 0) drain_wait(&bars[L::B_Q_FULL], (n_item - 1) & 1, lim);
      for (int st = 0; st < NK; ++st)
        if (kc > static_cast<uint32_t>(st)) {
          const uint32_t last = kc - 1 - ((kc - 1 - st) % NK);
          drain_wait(&bars[L::B_K_FULL + st], (last / NK) & 1, lim);
        }
      for (int st = 0; st < NV; ++st)
        if (vc > static_cast<uint32_t>(st)) {
          const uint32_t last = vc - 1 - ((vc - 1 - st) % NV);
          drain_wait(&bars[L::B_V_FULL + st], (last / NV) & 1, lim);
        }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, 0, 1);
      const uint32_t qaddr = smem_u32(sQ), kaddr = smem_u32(sK), vaddr = smem_u32(sV);
      uint32_t it = 0;
      int n_item = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total_items && ok; w += gridDim.x, ++n_item) {
        const WorkItem wi = decode_item(w, S, H, s_cu, s_order, s_istart);
        if (!mbar_wait(&bars[L::B_Q_FULL], n_item & 1, args.ctl, abort_flag)) break;
        // O += P V for global iteration c (first = first key tile of the item)
        auto issue_pv = [&](uint32_t c, bool first) -> bool {
          const int st = c % NV;
          const int b = c & 1;
          if (!mbar_wait(&bars[L::B_V_FULL + st], (c / NV) & 1, args.ctl, abort_flag)) return false;
          if (!mbar_wait(&bars[L::B_P_FULL + b], (c >> 1) & 1, args.ctl, abort_flag)) return false;
          if (first && !mbar_wait(&bars[L::B_O_EMPTY], (n_item & 1) ^ 1, args.ctl, abort_flag))
            return false;
          tc_fence_after();
          const uint32_t p_col = tmem + (b ? TM_P1 : TM_P0);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            // V tile: 16 key rows x D columns, MN-major, 128-byte swizzle;
            // LBO = distance between 64-column boxes, SBO = 8 rows of 128 B.
            const uint64_t bdesc =
                sdesc_sw128(vaddr + st * L::TILE_BYTES + kk * 16 * 128, BOX_BYTES, 1024);
            umma_ts(tmem + TM_O, p_col + kk * 8, bdesc, IDESC_PV, (first && kk == 0) ? 0u : 1u);
          }
          umma_commit(&bars[L::B_V_EMPTY + st]);
          umma_commit(&bars[L::B_PV_DONE + b]);
          return true;
        };
        for (int j = 0; j < wi.nkv && ok; ++j) {
          const uint32_t c = it + j;
          const int st = c % NK;
          const int b = c & 1;
          if (!mbar_wait(&bars[L::B_K_FULL + st], (c / NK) & 1, args.ctl, abort_flag)) { ok = false; break; }
          if (!mbar_wait(&bars[L::B_S_FREE + b], ((c >> 1) & 1) ^ 1, args.ctl, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t s_col = tmem + (b ? TM_S1 : TM_S0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            // Q and K tiles: K-major, 128-byte swizzle; a 16-element K step is a
            // 32-byte advance inside a 64-column box.
            const uint32_t koff = (kk >> 2) * BOX_BYTES + (kk & 3) * 32;
            const uint64_t adesc = sdesc_sw128(qaddr + koff, 16, 1024);
            const uint64_t bdesc = sdesc_sw128(kaddr + st * L::TILE_BYTES + koff, 16, 1024);
            umma_ss(s_col, adesc, bdesc, IDESC_S, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars[L::B_K_EMPTY + st]);
          umma_commit(&bars[L::B_S_FULL + b]);
          if (j == wi.nkv - 1) umma_commit(&bars[L::B_Q_EMPTY]);
          if (j > 0 && !issue_pv(c - 1, j == 1)) { ok = false; break; }
        }
        if (!ok) break;
        if (!issue_pv(it + wi.nkv - 1, wi.nkv == 1)) { ok = false; break; }
        umma_commit(&bars[L::B_O_FULL]);
        it += wi.nkv;
      }
      // every MMA this thread issued completes before TMEM is released
      umma_commit(&bars[L::B_DRAIN]);
      drain_wait(&bars[L::B_DRAIN], 0, args.ctl.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ============================================================ softmax + epilogue
    const int wq = warp & 3;          // TMEM sub-partition of this warp
    const int row = wq * 32 + lane;   // query row of this thread inside the tile
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const float scale_log2 = args.scale_log2;
    uint32_t it = 0;
    int n_item = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < total_items && ok; w += gridDim.x, ++n_item) {
      const WorkItem wi = decode_item(w, S, H, s_cu, s_order, s_istart);
      const int last_cols = wi.n - (wi.nkv - 1) * BN;  // valid keys in the last tile
      float m_ref = 0.f;  // reference max (scaled, log2 units)
      float l = 0.f;
      for (int j = 0; j < wi.nkv; ++j, ++it) {
        const int b = it & 1;
        if (!warp_wait(&bars[L::B_S_FULL + b], (it >> 1) & 1, args.ctl, abort_flag)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[128];
        const uint32_t s_addr = tmem + lane_base + (b ? TM_S1 : TM_S0);
        tmem_ld32(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[L::B_S_FREE + b]);
        float* sv = reinterpret_cast<float*>(sr);
        if (j == wi.nkv - 1 && last_cols < BN) {
#pragma unroll
          for (int cidx = 0; cidx < BN; ++cidx)
            if (cidx >= last_cols) sv[cidx] = -INFINITY;
        }
        float mx = sv[0];
#pragma unroll
        for (int cidx = 1; cidx < BN; ++cidx) mx = fmaxf(mx, sv[cidx]);
        const float m_tile = mx * scale_log2;
        if (j == 0) {
          m_ref = m_tile;
        } else if (m_tile > m_ref + RESCALE_THRESHOLD) {
          // O holds sum_j 2^(s' - m_ref) v_j: bring it to the new reference.
          const uint32_t cprev = it - 1;
          if (!warp_wait(&bars[L::B_PV_DONE + (cprev & 1)], (cprev >> 1) & 1, args.ctl, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float factor = ex2_approx(m_ref - m_tile);
          l *= factor;
#pragma unroll
          for (int cc = 0; cc < D; cc += 32) {
            uint32_t orr[32];
            tmem_ld32(tmem + lane_base + TM_O + cc, orr);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * factor);
            tmem_st32(tmem + lane_base + TM_O + cc, orr);
          }
          tmem_st_wait();
          m_ref = m_tile;
        }
        // P = 2^(s * scale * log2 e - m_ref), packed to bf16 pairs
        uint32_t pp[64];
        float lsum = 0.f;
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const float p0 = ex2_approx(fmaf(sv[2 * e], scale_log2, -m_ref));
          const float p1 = ex2_approx(fmaf(sv[2 * e + 1], scale_log2, -m_ref));
          lsum += p0 + p1;
          pp[e] = pack_bf16x2(p0, p1);
        }
        l += lsum;
        if (it >= 2) {  // PV of iteration it-2 has read this P buffer
          if (!warp_wait(&bars[L::B_PV_DONE + b], ((it >> 1) & 1) ^ 1, args.ctl, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        const uint32_t p_addr = tmem + lane_base + (b ? TM_P1 : TM_P0);
        tmem_st32(p_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&pp[0]));
        tmem_st32(p_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&pp[32]));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[L::B_P_FULL + b]);
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      if (!warp_wait(&bars[L::B_O_FULL], n_item & 1, args.ctl, abort_flag)) break;
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool row_valid = (wi.qt * BM + row) < wi.n;
      const int t = wi.row0 + row;
      uint32_t ov[D];
#pragma unroll
      for (int cc = 0; cc < D; cc += 32)
        tmem_ld32(tmem + lane_base + TM_O + cc, *reinterpret_cast<uint32_t(*)[32]>(&ov[cc]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[L::B_O_EMPTY]);
      if (row_valid) {
        if constexpr (GATED) {
          const int hid = H * D;
          const int m = __ldg(args.ep.tok_mod + t) ? 1 : 0;
          const float* gate =
              args.ep.mod + ((static_cast<size_t>(wi.s) * 2 + m) * 3 + 2) * hid + wi.h * D;
          const uint4* xr = reinterpret_cast<const uint4*>(args.ep.x + static_cast<size_t>(t) * hid + wi.h * D);
          uint4* yr = reinterpret_cast<uint4*>(args.ep.y + static_cast<size_t>(t) * hid + wi.h * D);
#pragma unroll
          for (int c8 = 0; c8 < D / 8; ++c8) {
            const uint4 xv = __ldg(xr + c8);
            const float4 g0 = __ldg(reinterpret_cast<const float4*>(gate + c8 * 8));
            const float4 g1 = __ldg(reinterpret_cast<const float4*>(gate + c8 * 8 + 4));
            const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
            uint32_t outw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = __uint_as_float(xw[e] << 16);
              const float x1 = __uint_as_float(xw[e] & 0xFFFF0000u);
              const float o0 = __uint_as_float(ov[c8 * 8 + 2 * e]) * inv_l;
              const float o1 = __uint_as_float(ov[c8 * 8 + 2 * e + 1]) * inv_l;
              outw[e] = pack_bf16x2(fmaf(gv[2 * e], o0, x0), fmaf(gv[2 * e + 1], o1, x1));
            }
            yr[c8] = make_uint4(outw[0], outw[1], outw[2], outw[3]);
          }
        } else {
          uint4* orow = reinterpret_cast<uint4*>(args.ep.o + (static_cast<size_t>(t) * H + wi.h) * D);
#pragma unroll
          for (int c8 = 0; c8 < D / 8; ++c8) {
            uint32_t outw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              outw[e] = pack_bf16x2(__uint_as_float(ov[c8 * 8 + 2 * e]) * inv_l,
                                    __uint_as_float(ov[c8 * 8 + 2 * e + 1]) * inv_l);
            orow[c8] = make_uint4(outw[0], outw[1], outw[2], outw[3]);
          }
        }
        if (args.ep.lse != nullptr)
          args.ep.lse[static_cast<size_t>(wi.h) * args.T + t] =
              (m_ref + __log2f(l)) * 0.69314718055994530942f;
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// Host-side tensor-map creation through the driver entry point (no link-time
// dependency on libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
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

// [T][H*D] bf16 viewed as a 2D tensor; box = 64 columns x 128 rows, 128-byte
// swizzle; rows past T read as zeros.
bool make_tile_map(CUtensorMap* map, const void* base, int32_t T, int32_t cols) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <int D, bool GATED>
cudaError_t launch_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const AttnArgs& a, int grid, cudaStream_t st) {
  constexpr int smem = Layout<D>::SMEM_BYTES;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(varlen_attn_kernel<D, GATED>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  varlen_attn_kernel<D, GATED><<<grid, NUM_THREADS, smem, st>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

int sm_count_dev() {
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

}  // namespace

cudaError_t launch_attention(const mf_bf16* q, const mf_bf16* k, const mf_bf16* v,
                             const int32_t* cu_seqlens_d, int32_t S, int32_t T, int32_t H,
                             int32_t D, float softmax_scale, const AttnEpilogue& ep,
                             int32_t num_items, const KernelCtl& ctl, cudaStream_t st) {
  if (num_items <= 0) return cudaSuccess;
  CUtensorMap mq, mk, mv;
  const int32_t cols = H * D;
  if (!make_tile_map(&mq, q, T, cols) || !make_tile_map(&mk, k, T, cols) ||
      !make_tile_map(&mv, v, T, cols))
    return cudaErrorInvalidValue;
  AttnArgs a;
  a.cu_seqlens = cu_seqlens_d;
  a.S = S;
  a.T = T;
  a.H = H;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.ep = ep;
  a.ctl = ctl;
  const int sms = sm_count_dev();
  const int grid = num_items < sms ? num_items : sms;
  const bool gated = ep.y != nullptr;
  if (D == 128) {
    return gated ? launch_t<128, true>(mq, mk, mv, a, grid, st)
                 : launch_t<128, false>(mq, mk, mv, a, grid, st);
  }
  if (D == 64) {
    return gated ? launch_t<64, true>(mq, mk, mv, a, grid, st)
                 : launch_t<64, false>(mq, mk, mv, a, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace mf
