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
// Design (one persistent CTA per SM, 12 warps). A work item is (sample, head,
// 256-row query block) = two 128-row query tiles A and B that share every K/V
// tile the CTA loads, which halves K/V traffic per FLOP and lets the softmax of
// one tile overlap the MMAs of the other:
//   warp 0      TMA producer: the item's Q tiles, then K and V tiles (128 keys)
//               of the item's own sample only, in separate 2-stage rings.
//   warp 1      tcgen05 issuer. Per key tile c, in this order:
//                 PV_A(c)  O_A += P_A V_c   (P_A read from TMEM as the A operand)
//                 S_A(c+1) = Q_A K_{c+1}^T  (overwrites S_A/P_A in TMEM)
//                 PV_B(c), S_B(c+1)
//               MMAs from one thread execute in issue order, so S_X(c+1) never
//               overwrites P_X(c) before PV_X(c) has read it, and the commit that
//               signals S_X(c+1) also covers PV_X(c).
//   warps 2..3  idle (they complete the first warpgroup, which gives most of its
//               registers to the softmax warpgroups with setmaxnreg).
//   warps 4..7  softmax + epilogue of tile A, one thread per query row (TMEM
//   warps 8..11 lane); the same for tile B. Online softmax in the exp2 domain:
//               the reference max is the first key tile's row max, and
//               exponentials of later tiles are taken against it as long as the
//               tile's row sum stays below 2^32 (which bounds every P); only
//               then is the reference moved to the tile max, O rescaled in TMEM
//               and the tile redone (exact after the final 1/l: a stale
//               reference scales numerator and denominator alike). P is packed
//               to bf16 into the first 64 columns of the tile's S region. With
//               RoPE fused, each thread first turns its own query row of the
//               item's Q tile in shared memory.
// RoPE in the load prologue ([rope]: per-sample 2D / 3D rotary embeddings; the
// pages name it among the fused operations of the block): q is read unrotated
// and every pair of a Q tile's row turns in shared memory by (cos, sin) looked
// up for the token's position in a small per-position table (one set of
// columns serves every axis), so no rotated copy of q reaches memory. The next
// item's Q tiles land in shared memory as the item's last S MMAs complete; the
// softmax warps turn them right after the item's last P if they have landed
// (else after the epilogue). K arrives
// rotated by a RoPE pass over k: a K tile is visited by every query block of
// its sample and head, and turning it at each visit (8192 pair rotations per
// tile by the two idle warps) measured 1.6x slower than the pass.
// TMEM (512 columns): S_A/P_A | S_B/P_B | O_A | O_B.
// Work items are ordered longest sample first and, inside a sample, the query
// blocks of one head next to each other so that concurrently running CTAs stream
// the same K/V tiles through L2. Key tiles start at the sample's first token and
// never leave the sample: tiles of other samples are never visited; only the
// last key tile of a sample can be partial and only it is masked.
//
// Every wait is bounded (mbar_wait); on expiry the CTA records MF_ERR_TIMEOUT,
// lets its in-flight copies and MMAs finish, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdint>
#include <functional>
#include <queue>
#include <utility>
#include <vector>

#include "mf_internal.h"
#include "mf_ptx.cuh"

namespace mf {

namespace {

constexpr int BM = 128;              // query rows per tile (MMA M)
constexpr int QB = 2 * BM;           // query rows per work item (tiles A and B)
constexpr int BN = 128;              // key rows per tile (MMA N of QK^T, K of PV)
constexpr int NUM_THREADS = 384;     // 3 warpgroups: {TMA, MMA, 2 idle}, softmax A, softmax B
// Registers: launched at 168 per thread (384 x 168 = 64512 of the 65536), then
// the first warpgroup gives up to 104 and the softmax warpgroups take 200 each:
// 128 * (104 + 200 + 200) = 64512, the launch's own total. 104 keeps the fully
// unrolled MMA issue (16 MMAs per key tile, issued back to back: measured 8%
// faster than a rolled loop) free of spills.
constexpr int kLaunchRegs = 168;
constexpr int kRegsControl = 104;
constexpr int kRegsSoftmax = 200;
static_assert(128 * (kRegsControl + 2 * kRegsSoftmax) <= NUM_THREADS * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr uint32_t kSoftmaxWarpsPerTile = 4;
constexpr uint32_t TMEM_COLS = 512;
// TMEM columns of tile x: S_X (fp32) with P_X (bf16x2) in its first 64 columns,
// and O_X (fp32, D columns)
__host__ __device__ constexpr uint32_t tm_s(int x) { return 128u * x; }
__host__ __device__ constexpr uint32_t tm_o(int x) { return 256u + 128u * x; }
constexpr int BOX_BYTES = 128 * 128;  // one TMA box: 128 rows x 64 bf16 (128 B), swizzled
constexpr int NK = 2;                 // K tile ring stages
constexpr int NV = 2;                 // V tile ring stages
// Of every 8 key pairs, this many are exponentiated on the FMA pipe
// (exp2_poly2) and the rest on the MUFU unit, which the two softmax warpgroups
// share. Measured on B200 (edit pack, attention alone, two runs each):
// 0 -> 1032, 1 -> 1053, 2 -> 1145 / 1084, 3 -> 1066 / 1002 useful TFLOP/s.
constexpr int kPolyPairsOf8 = 2;
// Redo bound on a tile's row sum (see the softmax loop).
constexpr float kRedoSum = 4294967296.f;  // 2^32


// Shared-memory layout. PAIR: the CTA is one of a cluster pair that runs M = 256
// MMAs together; it keeps its own 128 rows of each Q tile, half of each K tile's
// keys (64 rows) and half of each V tile's head dims (64 columns), and the
// smaller stages buy deeper K / V rings.
template <int D, bool PAIR>
struct Layout {
  static_assert(!PAIR || D == 128, "CTA pairs take head_dim 128 (a V half is one 128-byte box)");
  static constexpr int kBoxes = D / 64;  // 64-column boxes per Q / K row
  static constexpr int TILE_BYTES = BM * D * 2;           // one Q tile (this CTA's rows)
  static constexpr int NKS = PAIR ? 4 : NK;               // K ring stages
  static constexpr int NVS = PAIR ? 4 : NV;               // V ring stages
  static constexpr int K_ROWS = PAIR ? BN / 2 : BN;       // keys of a K tile held here
  static constexpr int K_BOX = K_ROWS * 128;              // one 64-column box of a K stage
  static constexpr int K_STAGE = K_ROWS * D * 2;
  static constexpr int V_COLS = PAIR ? D / 2 : D;         // head dims of a V tile held here
  static constexpr int V_STAGE = BN * V_COLS * 2;
  static constexpr uint32_t kPeers = PAIR ? 2 : 1;        // CTAs whose softmax warps arrive
  static constexpr int OFF_Q = 0;  // Q_A, Q_B
  static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + NKS * K_STAGE;
  static constexpr int OFF_BAR = OFF_V + NVS * V_STAGE;
  // barriers (arrival count 1 unless arrivals() says otherwise). With PAIR the
  // leader's FULL barriers of K and V count both CTAs' bytes, its Q_ROT, P_FULL
  // and O_EMPTY both CTAs' softmax warps; EMPTY, S_FULL and O_FULL arrive in
  // both CTAs from the leader's multicast commits.
  static constexpr int B_Q_FULL = 0;                 // [tile]
  static constexpr int B_Q_EMPTY = B_Q_FULL + 2;     // [tile]
  static constexpr int B_Q_ROT = B_Q_EMPTY + 2;      // [tile], one arrival per softmax warp
  static constexpr int B_K_FULL = B_Q_ROT + 2;       // NKS
  static constexpr int B_K_EMPTY = B_K_FULL + NKS;   // NKS
  static constexpr int B_V_FULL = B_K_EMPTY + NKS;   // NVS
  static constexpr int B_V_EMPTY = B_V_FULL + NVS;   // NVS
  static constexpr int B_S_FULL = B_V_EMPTY + NVS;   // [tile]
  static constexpr int B_P_FULL = B_S_FULL + 2;      // [tile], one arrival per softmax warp
  static constexpr int B_O_FULL = B_P_FULL + 2;      // [tile]
  static constexpr int B_O_EMPTY = B_O_FULL + 2;     // [tile], one arrival per softmax warp
  static constexpr int B_DRAIN = B_O_EMPTY + 2;
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
    if (i == B_P_FULL || i == B_P_FULL + 1 || i == B_O_EMPTY || i == B_O_EMPTY + 1 ||
        i == B_Q_ROT || i == B_Q_ROT + 1)
      return kSoftmaxWarpsPerTile * kPeers;
    return 1u;
  }
};

// Per-CTA work lists computed on the host (greedy longest-processing-time
// assignment), passed in the kernel parameters. CTA b runs ids[start[b]],
// ids[start[b] + 1], ... up to an entry of kSchedEnd. valid == 0 means "use the
// snake order" (too many items, or CTAs, for the table).
constexpr int kMaxSchedItems = 4096;
constexpr int kMaxSchedCtas = 160;
constexpr int32_t kSchedEnd = 0x7fffffff;
struct Schedule {
  int32_t valid;
  int32_t start[kMaxSchedCtas];
  int32_t ids[kMaxSchedItems + kMaxSchedCtas];  // items plus one end mark per CTA
};

// RoPE fused into the load prologue: pair i of axis a turns by the (cos, sin)
// at tab[pos_a][i] (one row of D / (2 axes) pairs per position; every axis
// uses the same frequencies).
struct AttnRope {
  const int32_t* pos_ids;  // [T][3] (f, h, w)
  const float2* tab;       // [P][D / (2 axes)]
  int32_t P;
};



struct AttnArgs {
  Schedule sched;
  const int32_t* cu_seqlens;
  int32_t S, T, H;
  float scale_log2;  // softmax_scale * log2(e)
  AttnEpilogue ep;
  AttnRope rope;
  KernelCtl ctl;
};

struct WorkItem {
  int32_t s, qb, h, row0, kv0, n, nkv;
  bool has_b;  // tile B holds at least one row of the sample
};

// A work item covers IQ query rows of one (sample, head): tiles A and B of
// IQ / 2 rows each (IQ = 256 for one CTA, 512 for a CTA pair, whose CTAs hold
// 128 rows of each tile).
template <int IQ>
__device__ __forceinline__ WorkItem decode_item(int w, int S, const int32_t* s_cu,
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
  const int nq = (it.n + IQ - 1) / IQ;
  it.h = local / nq;
  it.qb = local - it.h * nq;
  it.row0 = it.kv0 + it.qb * IQ;
  it.nkv = (it.n + BN - 1) / BN;
  it.has_b = (it.n - it.qb * IQ) > IQ / 2;
  return it;
}

// k-th work item of CTA b among G CTAs: rounds of G items in longest-first
// order, dealt forwards in even rounds and backwards in odd ones, which evens
// out the CTAs' totals when item sizes fall along the order. Every role of a CTA
// walks the same sequence.
__device__ __forceinline__ int snake_item(int k, int b, int G) {
  return k * G + ((k & 1) ? (G - 1 - b) : b);
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

// Rotates one row of a 128-row tile in shared memory (TMA layout: D / 64 boxes
// of 128 rows x 128 bytes, 16-byte chunks swizzled by row & 7) by the RoPE of
// the token at position (p0, p1, p2) = (f, h, w): pair (2i, 2i+1) turns by
// the angle whose (cos, sin) the table holds for the position on the pair's axis. The pair -> (axis, column) map
// is fixed by D and the axis count: every axis owns NPA = D / (2 AXES)
// consecutive pairs, in axis order (h, w) or (f, h, w); pairs past them stay.
// fp32 arithmetic, bf16 result, the same rounding as the standalone RoPE pass.
// G chunks (4G pairs) at a time: their shared-memory words and table entries
// are all requested before any is used. A position outside the table is
// recorded as MF_ERR_INVALID and leaves the row as it is.
template <int D, int AXES, int G>
__device__ __forceinline__ void rope_row_smem(uint8_t* tile, int row, int p0, int p1, int p2,
                                              const float2* tab, int P, const KernelCtl& ctl) {
  static_assert(AXES == 0 || AXES == 2 || AXES == 3, "RoPE axis count");
  if constexpr (AXES == 0) return;  // no RoPE: nothing to turn
  constexpr int NPA = D / (2 * (AXES == 0 ? 1 : AXES));  // pairs per axis (= table columns)
  constexpr int NCH = D / 8;           // 16-byte chunks per row
  static_assert(NCH % G == 0, "chunks per batch");
  if (static_cast<unsigned>(p0) >= static_cast<unsigned>(P) ||
      static_cast<unsigned>(p1) >= static_cast<unsigned>(P) ||
      static_cast<unsigned>(p2) >= static_cast<unsigned>(P)) {
    atomicCAS(ctl.err, 0, static_cast<int>(MF_ERR_INVALID));
    return;
  }
  // table rows of the axes in pair order: (h, w) for 2D, (f, h, w) for 3D
  const float2* rt[3] = {tab + static_cast<size_t>(AXES == 2 ? p1 : p0) * NPA,
                         tab + static_cast<size_t>(AXES == 2 ? p2 : p1) * NPA,
                         tab + static_cast<size_t>(p2) * NPA};
  uint8_t* rbase = tile + row * 128;
#pragma unroll
  for (int c0 = 0; c0 < NCH; c0 += G) {
    uint4* ptr[G];
    uint4 v[G];
    float2 cs[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int c = c0 + g;  // chunk in the head row: box c / 8, chunk c % 8 of the box
      ptr[g] = reinterpret_cast<uint4*>(rbase + (c >> 3) * BOX_BYTES +
                                        (((c & 7) ^ (row & 7)) << 4));
      v[g] = *ptr[g];
      if constexpr (NPA % 4 == 0) {
        // the chunk's four pairs share one axis and are four consecutive columns
        const int a = (4 * c) / NPA;
        if (a < AXES) {
          const float4* src = reinterpret_cast<const float4*>(rt[a] + (4 * c - a * NPA));
          const float4 lo = __ldg(src), hi = __ldg(src + 1);
          cs[g][0] = make_float2(lo.x, lo.y);
          cs[g][1] = make_float2(lo.z, lo.w);
          cs[g][2] = make_float2(hi.x, hi.y);
          cs[g][3] = make_float2(hi.z, hi.w);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int pr = 4 * c + e;
          const int a = pr / NPA;
          if (a < AXES) cs[g][e] = __ldg(rt[a] + (pr - a * NPA));
        }
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int c = c0 + g;
      uint32_t w[4] = {v[g].x, v[g].y, v[g].z, v[g].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int pr = 4 * c + e;
        if (pr / NPA < AXES) {
          const float x0 = __uint_as_float(w[e] << 16);
          const float x1 = __uint_as_float(w[e] & 0xFFFF0000u);
          w[e] = pack_bf16x2(x0 * cs[g][e].x - x1 * cs[g][e].y, x0 * cs[g][e].y + x1 * cs[g][e].x);
        }
      }
      *ptr[g] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// AXES: 0 = q and k arrive rotated; 2 or 3 = RoPE with that many axes fused
// into the Q load prologue (k arrives rotated).
template <int D, bool GATED, int AXES, bool PAIR>
// Registers are split per SM sub-partition: with 12 warps each sub-partition
// holds three, which caps a thread at 16384 / (3 * 32) = 170 -> 168 at launch.
// PAIR: launched in clusters of two CTAs (see Layout and the issuer below).
__global__ void __launch_bounds__(NUM_THREADS, 1)
    varlen_attn_kernel(const __grid_constant__ CUtensorMap tmap_q,
                       const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v,
                       const __grid_constant__ AttnArgs args) {
  using L = Layout<D, PAIR>;
  constexpr bool ROPE = AXES != 0;
  constexpr int IQ = PAIR ? 2 * QB : QB;  // query rows per work item
  constexpr int TQ = IQ / 2;              // rows per query tile (A or B), over the pair
  constexpr uint16_t kBoth = 3;           // multicast mask: both CTAs of the pair
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
    if constexpr (PAIR) {
      // both CTAs' warp 1, the same slot offset: the pair's TMEM at one address
      tmem_alloc_pair(tmem_slot, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int r = 0; r < S; ++r) {
      s_istart[r] = acc;
      const int n = s_cu[s_order[r] + 1] - s_cu[s_order[r]];
      acc += ((n + IQ - 1) / IQ) * H;
    }
    s_istart[S] = acc;
    if (*bad_flag) atomicCAS(args.ctl.err, 0, static_cast<int>(MF_ERR_INVALID));
  }
  __syncthreads();
  // Both CTAs' barriers are initialised before either CTA's arrivals, commits
  // or copies can reach the other's.
  if constexpr (PAIR) cluster_sync();
  const uint32_t tmem = *tmem_slot;
  const int total_items = *bad_flag ? 0 : s_istart[S];
  // With PAIR the pair is the scheduling unit and rank 1 takes the second
  // 128 rows of every tile; the leader (rank 0) issues the MMAs.
  const int rank = PAIR ? static_cast<int>(cluster_ctarank()) : 0;
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int n_units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  // k-th work item of this unit (at least total_items once the list is exhausted)
  auto item_k = [&](int k) -> int {
    return args.sched.valid ? args.sched.ids[args.sched.start[unit] + k]
                            : snake_item(k, unit, n_units);
  };
  auto decode = [&](int w) { return decode_item<IQ>(w, S, s_cu, s_order, s_istart); };
  // Arrival of a softmax warp on a barrier the MMA thread waits on: the
  // leader's, across the cluster for rank 1.
  auto arrive_to_issuer = [&](int b) {
    if constexpr (PAIR)
      mbar_arrive_cluster(cluster_addr(&bars[b], 0));
    else
      mbar_arrive(&bars[b]);
  };

  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;

  // Each role sets its register budget inside its own branch: code after a
  // join of differently budgeted paths is compiled for the smaller budget.
  if (warp < 4) {
  regs_dec<kRegsControl>();
  if (warp == 0) {
    // ============================================================ TMA producer
    // Order of loads: Q_A (and Q_B), K_0, then (K_{j+1}, V_j): the MMA warp
    // consumes S(j+1) before PV_B(j), so K runs one tile ahead of V.
    if (lane == 0) {
      uint32_t kc = 0, vc = 0;  // K / V tiles issued so far (global over items)
      uint32_t nq[2] = {0, 0};  // Q tiles issued per tile slot
      bool ok = true;
      // With PAIR this CTA copies its half of each K tile (keys rank * 64 ..
      // +64) and of each V tile (head dims rank * 64 .. +64); both halves
      // complete on the leader's FULL barrier, which the leader's producer
      // arms for both CTAs' bytes (a copy that lands first only takes the
      // barrier's byte count below zero for a while).
      auto load_k = [&](const WorkItem& wi, int j) -> bool {
        const int st = kc % L::NKS;
        if (!mbar_wait(&bars[L::B_K_EMPTY + st], ((kc / L::NKS) & 1) ^ 1, args.ctl, abort_flag))
          return false;
        uint8_t* dst = sK + st * L::K_STAGE;
        const int y = wi.kv0 + j * BN + rank * L::K_ROWS;
        if constexpr (PAIR) {
          if (rank == 0) mbar_expect_tx(&bars[L::B_K_FULL + st], 2 * L::K_STAGE);
          const uint32_t lb = cluster_addr(&bars[L::B_K_FULL + st], 0);
#pragma unroll
          for (int b = 0; b < L::kBoxes; ++b)
            tma_load_2d_pair(dst + b * L::K_BOX, &tmap_k, lb, wi.h * D + 64 * b, y);
        } else {
          mbar_expect_tx(&bars[L::B_K_FULL + st], L::K_STAGE);
#pragma unroll
          for (int b = 0; b < L::kBoxes; ++b)
            tma_load_2d(dst + b * L::K_BOX, &tmap_k, &bars[L::B_K_FULL + st], wi.h * D + 64 * b, y);
        }
        ++kc;
        return true;
      };
      auto load_v = [&](const WorkItem& wi, int j) -> bool {
        const int st = vc % L::NVS;
        if (!mbar_wait(&bars[L::B_V_EMPTY + st], ((vc / L::NVS) & 1) ^ 1, args.ctl, abort_flag))
          return false;
        uint8_t* dst = sV + st * L::V_STAGE;
        const int y = wi.kv0 + j * BN;
        if constexpr (PAIR) {
          if (rank == 0) mbar_expect_tx(&bars[L::B_V_FULL + st], 2 * L::V_STAGE);
          tma_load_2d_pair(dst, &tmap_v, cluster_addr(&bars[L::B_V_FULL + st], 0),
                           wi.h * D + rank * L::V_COLS, y);
        } else {
          mbar_expect_tx(&bars[L::B_V_FULL + st], L::V_STAGE);
#pragma unroll
          for (int b = 0; b < L::kBoxes; ++b)
            tma_load_2d(dst + b * BOX_BYTES, &tmap_v, &bars[L::B_V_FULL + st], wi.h * D + 64 * b, y);
        }
        ++vc;
        return true;
      };
      for (int k = 0, w = item_k(0); w < total_items && ok; w = item_k(++k)) {
        const WorkItem wi = decode(w);
        const int ntiles = wi.has_b ? 2 : 1;
        // each query tile has its own full / empty barriers, so the warps of
        // tile B only ever see the phases of items that hold a tile B
        for (int x = 0; x < ntiles && ok; ++x) {
          if (!mbar_wait(&bars[L::B_Q_EMPTY + x], (nq[x] & 1) ^ 1, args.ctl, abort_flag)) {
            ok = false;
            break;
          }
          // this CTA's own 128 rows of the tile, on its own barrier
          mbar_expect_tx(&bars[L::B_Q_FULL + x], L::TILE_BYTES);
#pragma unroll
          for (int b = 0; b < L::kBoxes; ++b)
            tma_load_2d(sQ + x * L::TILE_BYTES + b * BOX_BYTES, &tmap_q, &bars[L::B_Q_FULL + x],
                        wi.h * D + 64 * b, wi.row0 + x * TQ + rank * BM);
          ++nq[x];
        }
        if (!ok) break;
        if (!load_k(wi, 0)) break;
        for (int j = 0; j < wi.nkv; ++j) {
          if (j + 1 < wi.nkv && !load_k(wi, j + 1)) { ok = false; break; }
          if (!load_v(wi, j)) { ok = false; break; }
        }
      }
      // Let every copy this thread started land before the CTA can exit. With
      // PAIR, K and V copies complete on the leader's barriers: the leader
      // drains them for both CTAs, and the pair's closing cluster barrier keeps
      // rank 1 alive until then.
      const uint64_t lim = args.ctl.wait_limit_ns;
      for (int x = 0; x < 2; ++x)
        if (nq[x] > 0) drain_wait(&bars[L::B_Q_FULL + x], (nq[x] - 1) & 1, lim);
      if (rank == 0) {
        for (int st = 0; st < L::NKS; ++st)
          if (kc > static_cast<uint32_t>(st)) {
            const uint32_t last = kc - 1 - ((kc - 1 - st) % L::NKS);
            drain_wait(&bars[L::B_K_FULL + st], (last / L::NKS) & 1, lim);
          }
        for (int st = 0; st < L::NVS; ++st)
          if (vc > static_cast<uint32_t>(st)) {
            const uint32_t last = vc - 1 - ((vc - 1 - st) % L::NVS);
            drain_wait(&bars[L::B_V_FULL + st], (last / L::NVS) & 1, lim);
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    // With PAIR only the leader issues: every MMA is M = 256 over the pair
    // (rank 0's 128 query rows, then rank 1's), B taken half from each CTA's
    // shared memory (S: 64 keys each; PV: 64 head dims each), and every commit
    // that a CTA's producer or softmax warps wait on is multicast to both.
    if (lane == 0 && rank == 0) {
      constexpr int MM = PAIR ? 2 * BM : BM;
      constexpr uint32_t IDESC_S = idesc_bf16_f32(MM, BN, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(MM, D, 0, 1);
      const uint32_t qaddr = smem_u32(sQ), kaddr = smem_u32(sK), vaddr = smem_u32(sV);
      uint32_t kv = 0;           // key tiles consumed so far (global over items)
      uint32_t itx[2] = {0, 0};  // tiles processed per query tile slot (global)
      int nit[2] = {0, 0};       // items processed per query tile slot
      bool ok = true;
      // with RoPE fused, a Q tile is ready once its softmax warps have turned
      // it, and with PAIR once both CTAs' softmax warps have seen their rows
      // land; otherwise once its copy has landed (K always arrives rotated)
      constexpr int kQReady = (ROPE || PAIR) ? L::B_Q_ROT : L::B_Q_FULL;
      constexpr int kKReady = L::B_K_FULL;
      auto commit = [&](int b) {
        if constexpr (PAIR)
          umma_commit_pair(&bars[b], kBoth);
        else
          umma_commit(&bars[b]);
      };
      // Shared-memory descriptors are built once per operand base; a byte offset
      // o inside shared memory moves the start-address field by o >> 4 (the
      // field cannot carry: shared addresses stay below 256 KB).
      const uint64_t qdesc = sdesc_sw128(qaddr, 16, 1024);
      const uint64_t kdesc = sdesc_sw128(kaddr, 16, 1024);
      const uint64_t vdesc = sdesc_sw128(vaddr, BOX_BYTES, 1024);
      // S_X(c) = Q_X K_c^T into S_X; K-major operands, 128-byte swizzle; a
      // 16-element K step is a 32-byte advance inside a 64-column box.
      auto issue_s = [&](int x, uint32_t c) {
        const uint64_t a0 = qdesc + static_cast<uint64_t>((x * L::TILE_BYTES) >> 4);
        const uint64_t b0 = kdesc + static_cast<uint64_t>(((c % L::NKS) * L::K_STAGE) >> 4);
        const uint32_t d = tmem + tm_s(x);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t aoff = ((kk >> 2) * BOX_BYTES + (kk & 3) * 32) >> 4;
          const uint32_t boff = ((kk >> 2) * L::K_BOX + (kk & 3) * 32) >> 4;
          if constexpr (PAIR)
            umma_ss_pair(d, a0 + aoff, b0 + boff, IDESC_S, kk > 0 ? 1u : 0u);
          else
            umma_ss(d, a0 + aoff, b0 + boff, IDESC_S, kk > 0 ? 1u : 0u);
        }
        commit(L::B_S_FULL + x);
      };
      // O_X += P_X V_c; V is MN-major (LBO = distance between 64-column boxes,
      // SBO = 8 rows of 128 B); P_X comes from TMEM, 8 columns per 16 keys.
      auto issue_pv = [&](int x, uint32_t c, bool first) {
        const uint64_t b0 = vdesc + static_cast<uint64_t>(((c % L::NVS) * L::V_STAGE) >> 4);
        const uint32_t d = tmem + tm_o(x);
        const uint32_t a = tmem + tm_s(x);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t acc = (first && kk == 0) ? 0u : 1u;
          if constexpr (PAIR)
            umma_ts_pair(d, a + kk * 8, b0 + ((kk * 16 * 128) >> 4), IDESC_PV, acc);
          else
            umma_ts(d, a + kk * 8, b0 + ((kk * 16 * 128) >> 4), IDESC_PV, acc);
        }
      };
      auto wait = [&](int bar, uint32_t parity) -> bool {
        return mbar_wait(&bars[bar], parity, args.ctl, abort_flag);
      };
      for (int k = 0, w = item_k(0); w < total_items && ok; w = item_k(++k)) {
        const WorkItem wi = decode(w);
        const int ntiles = wi.has_b ? 2 : 1;
        // prologue: S_A(0), S_B(0)
        if (!wait(kKReady + kv % L::NKS, (kv / L::NKS) & 1)) break;
        for (int x = 0; x < ntiles && ok; ++x) {
          if (!wait(kQReady + x, nit[x] & 1)) { ok = false; break; }
          tc_fence_after();
          issue_s(x, kv);
        }
        if (!ok) break;
        commit(L::B_K_EMPTY + kv % L::NKS);
        if (wi.nkv == 1)
          for (int x = 0; x < ntiles; ++x) commit(L::B_Q_EMPTY + x);
        for (int j = 0; j < wi.nkv && ok; ++j) {
          const uint32_t c = kv + j;
          const bool more = j + 1 < wi.nkv;
          if (!wait(L::B_V_FULL + c % L::NVS, (c / L::NVS) & 1)) { ok = false; break; }
          if (more && !wait(kKReady + (c + 1) % L::NKS, ((c + 1) / L::NKS) & 1)) {
            ok = false;
            break;
          }
          for (int x = 0; x < ntiles; ++x) {
            // PV_X(j) once softmax X has written P_X(j) (and, on the item's first
            // tile, once the previous item's epilogue has read O_X)
            if (!wait(L::B_P_FULL + x, (itx[x] + j) & 1)) { ok = false; break; }
            if (j == 0 && !wait(L::B_O_EMPTY + x, (nit[x] & 1) ^ 1)) { ok = false; break; }
            tc_fence_after();
            issue_pv(x, c, j == 0);
            if (more) issue_s(x, c + 1);
          }
          if (!ok) break;
          commit(L::B_V_EMPTY + c % L::NVS);
          if (more) {
            commit(L::B_K_EMPTY + (c + 1) % L::NKS);
            if (j + 2 == wi.nkv)
              for (int x = 0; x < ntiles; ++x) commit(L::B_Q_EMPTY + x);
          }
        }
        if (!ok) break;
        for (int x = 0; x < ntiles; ++x) {
          commit(L::B_O_FULL + x);
          itx[x] += wi.nkv;
          ++nit[x];
        }
        kv += wi.nkv;
      }
      // every MMA this thread issued completes before TMEM is released
      if constexpr (PAIR)
        umma_commit_pair(&bars[L::B_DRAIN], 1);  // the leader's own barrier
      else
        umma_commit(&bars[L::B_DRAIN]);
      drain_wait(&bars[L::B_DRAIN], 0, args.ctl.wait_limit_ns);
    }
    __syncwarp();
  }
  } else {
    regs_inc<kRegsSoftmax>();
    // ============================================================ softmax + epilogue
    const int x = (warp - 4) >> 2;    // query tile: 0 = A (warps 4-7), 1 = B (warps 8-11)
    const int wq = warp & 3;          // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;   // query row inside the tile
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t s_col = tmem + lane_base + tm_s(x);
    const uint32_t o_col = tmem + lane_base + tm_o(x);
    const float scale_log2 = args.scale_log2;
    uint32_t it = 0;  // tiles of this query tile slot processed (global)
    int n_item = 0;   // items with this tile present
    bool ok = true;
    bool q_turned = false;  // this warp has already turned its rows of the item's Q tile
    // RoPE in the load prologue: this thread's query row of tile X, turned in
    // place once its copy has landed; the MMA warp issues S_X(0) once all four
    // warps of the tile have arrived on Q_ROT[X]
    // With PAIR (no RoPE) the same path only reports the landed copy: the
    // leader's MMA thread cannot see rank 1's copy barrier.
    auto turn_q = [&](const WorkItem& q_it) {
      if constexpr (ROPE) {
        const int rr = q_it.qb * IQ + x * TQ + rank * BM + row;  // row in the sample
        if (rr < q_it.n) {
          const int32_t* pp = args.rope.pos_ids + 3 * static_cast<size_t>(q_it.kv0 + rr);
          rope_row_smem<D, AXES, 8>(sQ + x * L::TILE_BYTES, row, __ldg(pp), __ldg(pp + 1),
                                    __ldg(pp + 2), args.rope.tab, args.rope.P, args.ctl);
        }
        fence_proxy_async_smem();  // the MMA reads the tile through the async proxy
      }
      __syncwarp();
      if (lane == 0) arrive_to_issuer(L::B_Q_ROT + x);
    };
    for (int k = 0, w = item_k(0); w < total_items && ok; w = item_k(++k)) {
      const WorkItem wi = decode(w);
      if (x == 1 && !wi.has_b) continue;
      if constexpr (ROPE || PAIR) {
        if (!q_turned) {
          if (!warp_wait(&bars[L::B_Q_FULL + x], n_item & 1, args.ctl, abort_flag)) break;
          turn_q(wi);
        }
        q_turned = false;
      }
      const int last_cols = wi.n - (wi.nkv - 1) * BN;  // valid keys in the last tile
      float m_ref = 0.f;  // reference max (scaled, log2 units)
      float l = 0.f;
      for (int j = 0; j < wi.nkv; ++j, ++it) {
        if (!warp_wait(&bars[L::B_S_FULL + x], it & 1, args.ctl, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const bool masked = (j == wi.nkv - 1) && (last_cols < BN);
        // scores of this row from TMEM (fp32), masked past the sample's end
        auto load_scores = [&](uint32_t (&sr)[BN]) {
#pragma unroll
          for (int cc = 0; cc < BN; cc += 32)
            tmem_ld32(s_col + cc, *reinterpret_cast<uint32_t(*)[32]>(&sr[cc]));
          tmem_ld_wait();
          if (masked) {
#pragma unroll
            for (int cidx = 0; cidx < BN; ++cidx)
              if (cidx >= last_cols) sr[cidx] = __float_as_uint(-INFINITY);
          }
        };
        // P = 2^(s * scale * log2 e - m_ref) for the row's 128 keys, packed to 64
        // bf16 pairs; the row sum goes to four packed fp32 accumulators. Per key
        // pair: one packed FMA, two ex2, one bf16 pack, one packed add.
        const uint64_t scale2 = f2_pack(scale_log2, scale_log2);
        auto exponentiate = [&](const uint32_t (&sr)[BN], uint32_t (&pp)[BN / 2], uint64_t (&ls)[4]) {
          const uint64_t neg_m2 = f2_pack(-m_ref, -m_ref);
#pragma unroll
          for (int e = 0; e < BN / 2; ++e) {
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])),
                                       scale2, neg_m2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            float p0, p1;
            if ((e % 8) < kPolyPairsOf8) {
              exp2_poly2(x0, x1, p0, p1);
            } else {
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
            }
            pp[e] = pack_bf16x2(p0, p1);
            ls[e & 3] = f2_add(ls[e & 3], f2_pack(p0, p1));
          }
        };
        // row max of a tile's scores (scaled to log2 units)
        auto tile_max = [&](const uint32_t (&sr)[BN]) -> float {
          float m4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) m4[e] = __uint_as_float(sr[e]);
#pragma unroll
          for (int cidx = 4; cidx < BN - 4; cidx += 8)
#pragma unroll
            for (int e = 0; e < 4; ++e)
              m4[e] = max3f(m4[e], __uint_as_float(sr[cidx + e]), __uint_as_float(sr[cidx + 4 + e]));
#pragma unroll
          for (int e = 0; e < 4; ++e) m4[e] = fmaxf(m4[e], __uint_as_float(sr[BN - 4 + e]));
          return fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * scale_log2;
        };
        auto row_sum = [](const uint64_t (&ls)[4]) -> float {
          float a0, a1, b0, b1, c0, c1, d0, d1;
          f2_unpack(ls[0], a0, a1);
          f2_unpack(ls[1], b0, b1);
          f2_unpack(ls[2], c0, c1);
          f2_unpack(ls[3], d0, d1);
          return ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
        };
        uint32_t pp[BN / 2];
        uint64_t ls[4] = {0, 0, 0, 0};  // packed (0.f, 0.f)
        {
          uint32_t sr[BN];
          load_scores(sr);
          if (j == 0) m_ref = tile_max(sr);  // first tile of the item: the reference is its max
          exponentiate(sr, pp, ls);
        }
        // A tile row sum above 2^32 (or inf / NaN) means some P may be out of
        // range: the max grew by more than 2^25 over the reference. Move the
        // reference to the tile max, bring O and l along (PV_X(j-1) is complete:
        // S_X(j) was issued after it) and redo the tile from the scores, still in
        // TMEM. Below the bound every P <= 2^32 and O, l stay far from overflow.
        // The TMEM loads and stores below are warp-collective (.sync.aligned), so
        // the whole warp takes the branch when any row needs it; for the other
        // rows moving the reference up to their own tile max is just as exact.
        float tile_sum = row_sum(ls);
        if (__any_sync(0xffffffffu, !(tile_sum <= kRedoSum))) {
          uint32_t sr2[BN];
          load_scores(sr2);
          const float m_new = fmaxf(m_ref, tile_max(sr2));
          const float factor = ex2_approx(m_ref - m_new);
          l *= factor;
#pragma unroll 1
          for (int cc = 0; cc < D; cc += 32) {
            uint32_t orr[32];
            tmem_ld32(o_col + cc, orr);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * factor);
            tmem_st32(o_col + cc, orr);
          }
          tmem_st_wait();
          m_ref = m_new;
#pragma unroll
          for (int e = 0; e < 4; ++e) ls[e] = 0;
          exponentiate(sr2, pp, ls);
          tile_sum = row_sum(ls);
        }
        l += tile_sum;
        tmem_st32(s_col + 0, *reinterpret_cast<uint32_t(*)[32]>(&pp[0]));
        tmem_st32(s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&pp[32]));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_to_issuer(L::B_P_FULL + x);
      }
      if (!ok) break;
      if constexpr (ROPE || PAIR) {
        // The next item's Q tile was requested when S_X(last) completed and has
        // often landed by now: turn it while PV_X(last) runs, so that S_X(0) of
        // the next item is computed during this epilogue rather than after it.
        // Only when the next item of this CTA holds tile X (then its copy is the
        // next phase of Q_FULL[X]), and only if every lane of the warp sees the
        // copy complete (each lane then has its own acquire); otherwise the tile
        // is turned after the epilogue.
        const int wn = item_k(k + 1);
        if (wn < total_items) {
          const WorkItem nx = decode(wn);
          if ((x == 0 || nx.has_b) &&
              __all_sync(0xffffffffu, mbar_try_wait(&bars[L::B_Q_FULL + x], (n_item + 1) & 1))) {
            turn_q(nx);
            q_turned = true;
          }
        }
      }
      // ---------------------------------------------------------- epilogue
      // O row in chunks of 32 columns: normalise by 1/l and write (y = x + gate
      // * O in the fused block, else O); then release O_X to the next item.
      const int r_in_sample = wi.qb * IQ + x * TQ + rank * BM + row;
      const int t = wi.row0 + x * TQ + rank * BM + row;
      const bool row_valid = r_in_sample < wi.n;
      const int col0 = wi.h * D;  // first column of this head in [T][H*D]
      const int hid = H * D;
      const float* gate = nullptr;
      // the block input row (the epilogue's only DRAM read) is requested before
      // waiting for the last PV, so its latency overlaps that MMA
      uint4 xv[GATED ? D / 8 : 1];
      if constexpr (GATED) {
        const int m = row_valid ? (__ldg(args.ep.tok_mod + t) ? 1 : 0) : 0;
        gate = args.ep.mod + ((static_cast<size_t>(wi.s) * 2 + m) * 3 + 2) * hid + col0;
        const uint4* xr = reinterpret_cast<const uint4*>(args.ep.x + static_cast<size_t>(t) * hid + col0);
#pragma unroll
        for (int c8 = 0; c8 < D / 8; ++c8) xv[c8] = row_valid ? __ldg(xr + c8) : make_uint4(0, 0, 0, 0);
      }
      if (!warp_wait(&bars[L::B_O_FULL + x], n_item & 1, args.ctl, abort_flag)) break;
      tc_fence_after();
      const float inv_l = 1.f / l;
#pragma unroll
      for (int cc = 0; cc < D; cc += 32) {
        uint32_t ov[32];
        tmem_ld32(o_col + cc, ov);
        tmem_ld_wait();
        if (row_valid) {
          if constexpr (GATED) {
            uint4* yr = reinterpret_cast<uint4*>(args.ep.y + static_cast<size_t>(t) * hid + col0 + cc);
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
              const uint4 xc = xv[cc / 8 + c8];
              const float4 g0 = __ldg(reinterpret_cast<const float4*>(gate + cc + c8 * 8));
              const float4 g1 = __ldg(reinterpret_cast<const float4*>(gate + cc + c8 * 8 + 4));
              const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
              const uint32_t xw[4] = {xc.x, xc.y, xc.z, xc.w};
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
            uint4* orow =
                reinterpret_cast<uint4*>(args.ep.o + static_cast<size_t>(t) * hid + col0 + cc);
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
              uint32_t outw[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                outw[e] = pack_bf16x2(__uint_as_float(ov[c8 * 8 + 2 * e]) * inv_l,
                                      __uint_as_float(ov[c8 * 8 + 2 * e + 1]) * inv_l);
              orow[c8] = make_uint4(outw[0], outw[1], outw[2], outw[3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_to_issuer(L::B_O_EMPTY + x);
      ++n_item;
      if (row_valid && args.ep.lse != nullptr)
        args.ep.lse[static_cast<size_t>(wi.h) * args.T + t] =
            (m_ref + __log2f(l)) * 0.69314718055994530942f;
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if constexpr (PAIR) {
    // The leader has drained its MMAs (which write rank 1's TMEM) and the
    // copies that complete on its barriers; neither CTA frees TMEM or leaves
    // before both are here.
    cluster_sync();
    if (warp == 1) tmem_dealloc_pair(tmem, TMEM_COLS);
  } else {
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
  }
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

// [T][H*D] bf16 viewed as a 2D tensor; box = 64 columns x box_rows rows,
// 128-byte swizzle; rows past T read as zeros.
bool make_tile_map(CUtensorMap* map, const void* base, int32_t T, int32_t cols,
                   uint32_t box_rows = 128) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <int D, bool GATED, int AXES, bool PAIR>
bool kernel_ready(int dev) {
  static bool attr_set[64] = {false};
  if (dev < 0 || dev >= 64) return false;
  if (!attr_set[dev]) {
    // The setmaxnreg split assumes the kernel was built with exactly
    // kLaunchRegs registers per thread; with fewer the softmax warpgroups'
    // setmaxnreg.inc could never be satisfied, so refuse to launch.
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, varlen_attn_kernel<D, GATED, AXES, PAIR>) != cudaSuccess ||
        fa.numRegs != kLaunchRegs)
      return false;
    if (cudaFuncSetAttribute(varlen_attn_kernel<D, GATED, AXES, PAIR>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Layout<D, PAIR>::SMEM_BYTES) != cudaSuccess)
      return false;
    attr_set[dev] = true;
  }
  return true;
}

template <int D, bool GATED, int AXES>
cudaError_t launch_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const AttnArgs& a, int grid, cudaStream_t st) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (!kernel_ready<D, GATED, AXES, false>(dev)) return cudaErrorInvalidConfiguration;
  varlen_attn_kernel<D, GATED, AXES, false>
      <<<grid, NUM_THREADS, Layout<D, false>::SMEM_BYTES, st>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

// CTA pairs: clusters of two, `pairs` of them (grid = 2 * pairs).
template <int D, bool GATED, int AXES>
cudaError_t launch_pair_t(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          const AttnArgs& a, int pairs, cudaStream_t st) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (!kernel_ready<D, GATED, AXES, true>(dev)) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = Layout<D, true>::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, varlen_attn_kernel<D, GATED, AXES, true>, mq, mk, mv, a);
}

// How many CTA pairs of the pair kernel can be resident at once (one CTA per
// SM, both CTAs of a pair in one GPC); cached per device.
template <bool GATED, int AXES>
int max_pairs(int dev) {
  static int cached[64] = {0};
  if (dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    if (!kernel_ready<128, GATED, AXES, true>(dev)) return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = Layout<128, true>::SMEM_BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, varlen_attn_kernel<128, GATED, AXES, true>, &cfg) !=
            cudaSuccess ||
        n <= 0)
      return 0;
    cached[dev] = n;
  }
  return cached[dev];
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

// Greedy longest-processing-time schedule over the items in the kernel's own
// numbering (samples longest first, ties by pack order; inside a sample
// item = head * query_blocks + query_block). An item over nkv key tiles costs
// nkv + 1 periods whether it holds one query tile or two: a lone tile's softmax
// is not hidden behind a second tile's MMAs, and timing showed it nearly as
// slow. Each item goes to the least-loaded CTA (lowest index on ties). The table is used only when this
// beats the snake order's estimated makespan by more than 1%: where the two
// tie (equal items, or one item per CTA) the snake order measured a little
// faster. Leaves s->valid = 0 for the snake order, and when the table cannot
// hold the items.
void build_schedule(const int32_t* cu_h, int32_t S, int32_t H, int grid, int iq, Schedule* s) {
  s->valid = 0;
  std::vector<int> order(S);
  for (int i = 0; i < S; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
    return (cu_h[a + 1] - cu_h[a]) > (cu_h[b + 1] - cu_h[b]);
  });
  int64_t total = 0;
  for (int i = 0; i < S; ++i) total += static_cast<int64_t>((cu_h[i + 1] - cu_h[i] + iq - 1) / iq) * H;
  if (total > kMaxSchedItems || grid > kMaxSchedCtas || grid <= 0) return;
  std::vector<std::vector<int32_t>> lists(grid);
  std::vector<int64_t> snake_load(grid, 0);
  using Slot = std::pair<int64_t, int>;  // (load, cta)
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
  for (int b = 0; b < grid; ++b) heap.push({0, b});
  int64_t greedy_max = 0;
  int32_t id = 0;
  for (int r = 0; r < S; ++r) {
    const int n = cu_h[order[r] + 1] - cu_h[order[r]];
    const int nq = (n + iq - 1) / iq;
    const int64_t nkv = (n + BN - 1) / BN;
    for (int h = 0; h < H; ++h) {
      for (int qb = 0; qb < nq; ++qb, ++id) {
        const int64_t cost = nkv + 1;
        const int k = id / grid, i = id - k * grid;
        snake_load[(k & 1) ? grid - 1 - i : i] += cost;
        Slot sl = heap.top();
        heap.pop();
        lists[sl.second].push_back(id);
        sl.first += cost;
        greedy_max = std::max(greedy_max, sl.first);
        heap.push(sl);
      }
    }
  }
  const int64_t snake_max = *std::max_element(snake_load.begin(), snake_load.end());
  if (greedy_max * 100 >= snake_max * 99) return;
  int32_t pos = 0;
  for (int b = 0; b < grid; ++b) {
    s->start[b] = pos;
    for (int32_t v : lists[b]) s->ids[pos++] = v;
    s->ids[pos++] = kSchedEnd;
  }
  s->valid = 1;
}

}  // namespace

int32_t attention_work_items(const int32_t* cu_h, int32_t S, int32_t H, bool pair) {
  const int64_t iq = pair ? 2 * QB : QB;
  int64_t n = 0;
  for (int32_t s = 0; s < S; ++s) n += (static_cast<int64_t>(cu_h[s + 1] - cu_h[s]) + iq - 1) / iq;
  return static_cast<int32_t>(n * H);
}

cudaError_t launch_attention(const mf_bf16* q, const mf_bf16* k, const mf_bf16* v,
                             const int32_t* cu_seqlens_d, const int32_t* cu_seqlens_h, int32_t S,
                             int32_t T, int32_t H, int32_t D, float softmax_scale,
                             const AttnEpilogue& ep, const AttnRopeParams* rope, bool pair,
                             const KernelCtl& ctl, cudaStream_t st) {
  const bool use_pair = pair && D == 128;  // CTA pairs take head_dim 128 only
  const int32_t num_items = attention_work_items(cu_seqlens_h, S, H, use_pair);
  if (num_items <= 0) return cudaSuccess;
  CUtensorMap mq, mk, mv;
  const int32_t cols = H * D;
  // a CTA of a pair copies 64 keys of each K tile
  if (!make_tile_map(&mq, q, T, cols) || !make_tile_map(&mk, k, T, cols, use_pair ? 64 : 128) ||
      !make_tile_map(&mv, v, T, cols))
    return cudaErrorInvalidValue;
  static thread_local AttnArgs a;  // ~17 KB: kept off the host stack
  a.cu_seqlens = cu_seqlens_d;
  a.S = S;
  a.T = T;
  a.H = H;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.ep = ep;
  a.ctl = ctl;
  a.rope = AttnRope{};
  if (rope != nullptr) {
    if (rope->axes != 2 && rope->axes != 3) return cudaErrorInvalidValue;
    a.rope.pos_ids = rope->pos_ids;
    a.rope.tab = reinterpret_cast<const float2*>(rope->tab);
    a.rope.P = rope->P;
  }
  const bool gated = ep.y != nullptr;
  // the fused gated residual is only used by the block, which always rotates
  if (gated && rope == nullptr) return cudaErrorInvalidValue;
  const int axes = rope ? rope->axes : 0;
  if (use_pair) {
    int dev = 0;
    cudaGetDevice(&dev);
    int mp = 0;
    if (axes == 0) mp = max_pairs<false, 0>(dev);
    else if (axes == 2) mp = gated ? max_pairs<true, 2>(dev) : max_pairs<false, 2>(dev);
    else mp = gated ? max_pairs<true, 3>(dev) : max_pairs<false, 3>(dev);
    if (mp <= 0) return cudaErrorInvalidConfiguration;
    const int pairs = num_items < mp ? num_items : mp;
    build_schedule(cu_seqlens_h, S, H, pairs, 2 * QB, &a.sched);
    if (axes == 0) return launch_pair_t<128, false, 0>(mq, mk, mv, a, pairs, st);
    if (axes == 2)
      return gated ? launch_pair_t<128, true, 2>(mq, mk, mv, a, pairs, st)
                   : launch_pair_t<128, false, 2>(mq, mk, mv, a, pairs, st);
    return gated ? launch_pair_t<128, true, 3>(mq, mk, mv, a, pairs, st)
                 : launch_pair_t<128, false, 3>(mq, mk, mv, a, pairs, st);
  }
  const int sms = sm_count_dev();
  const int grid = num_items < sms ? num_items : sms;
  build_schedule(cu_seqlens_h, S, H, grid, QB, &a.sched);
#define MF_ATTN_CASE(DD)                                                                   \
  if (D == DD) {                                                                           \
    if (axes == 0) return launch_t<DD, false, 0>(mq, mk, mv, a, grid, st);                 \
    if (axes == 2)                                                                         \
      return gated ? launch_t<DD, true, 2>(mq, mk, mv, a, grid, st)                        \
                   : launch_t<DD, false, 2>(mq, mk, mv, a, grid, st);                      \
    return gated ? launch_t<DD, true, 3>(mq, mk, mv, a, grid, st)                          \
                 : launch_t<DD, false, 3>(mq, mk, mv, a, grid, st);                        \
  }
  MF_ATTN_CASE(128)
  MF_ATTN_CASE(64)
#undef MF_ATTN_CASE
  return cudaErrorInvalidValue;
}

}  // namespace mf
