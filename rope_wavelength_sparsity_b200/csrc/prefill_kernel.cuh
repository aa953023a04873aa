// Windowed causal attention prefill for sm_100a (TMA + tcgen05 + TMEM).
//
// "ATFlash: Per-RoPE-Wavelength Attention Windows", Abstract: the window is a
// slice of the query-key contraction axis and the online-softmax recurrence
// is left untouched.  "WavePrune", Original abstract and summary: head dims
// are grouped in blocks of 16 so the pruned contraction still runs on the
// Tensor Cores.
//
// One CTA owns two 128-row query tiles (256 consecutive rows) of one
// (batch, query head); both walk the same key tiles from the diagonal
// outwards, so every K and V tile is loaded once for 256 rows.  Warp roles:
//   warps 0-3, 4-7  softmax of query tile 0 / 1: row r of a tile is TMEM lane
//              r.  They correct the pairs that are kept at some but not all
//              distances of the tile (adding those left out of the
//              contraction, subtracting those contracted but pruned), read S
//              from TMEM, mask, run the online softmax with a lazily rescaled
//              O, write P (bf16) back into TMEM over S, and finish with O / l.
//              The two groups alternate with the tensor core (ping-pong).
//   warp 8     TMA producer: both Q tiles once, then K and V tiles into a ring.
//   warp 9     MMA issuer (one lane): S_t = Q_t K^T over the active k-steps,
//              O_t += P_t V with P_t read from TMEM; owns the TMEM allocation.
//   warps 10-11 idle (they complete warpgroup 2 for the register hand-over).
//
// Shared-memory layouts.  Q and K use the no-swizzle canonical K-major layout
// with one 16-byte column panel per 8 head dims: panel c holds dims
// [8c, 8c+8) of all 128 rows (row r at byte 16 r), panels are 2 KB apart.
// A K=16 MMA step reads two core-matrix columns that are LBO bytes apart, so
// with LBO = (D/16) * 2 KB the step m pairs panel m (dims 8m..8m+7, the first
// halves of pairs 8m..8m+7) with panel D/16 + m (their second halves): every
// k-step carries 8 whole RoPE pairs, and skipping steps below k0 drops exactly
// the pairs 0 .. 8*k0 - 1.  V uses the 128-byte-swizzled MN-major layout
// (64-dim panels of 128 keys).
//
// TMEM columns: S_0 / P_0 at [0,128), S_1 / P_1 at [128,256), O_0 at
// [256, 256+D), O_1 at [256+D, 256+2D).  P_t (bf16 pairs) overwrites the
// first 64 columns of S_t; the next QK of tile t is issued after PV_t, and
// tcgen05 MMAs of one thread run in issue order.
//
// Grid.  One CTA per work item (a 256-row query block of one head of one
// sequence), heaviest query blocks first: one head after another, or, for
// g = 8 when K and V fit in L2, every head's heaviest blocks before any
// head's lighter ones.  The SPLIT instantiation runs work items as several
// CTAs over disjoint key ranges, each writing a partial result that
// prefill_combine_kernel merges; the host uses it for the items of a grid's
// last partial wave when all items do the same work.
#pragma once

#include "device_util.cuh"

namespace wpattn {

constexpr int kBM = 128;              // query rows per tile (TMEM lanes)
constexpr int kCT = 16;               // pairs per batch of the per-warp K transpose (g = 1)

// Tile shape.  TMEM (128 lanes x 512 columns) holds, per query tile, S (BN
// fp32 columns) and O (D columns).  Two query tiles on 128-key tiles fit
// both head dims (2 x (128 + 128) = 512 columns at D = 128).  The kernel
// also supports three query tiles on 96-key tiles (3 x (96 + 64) = 480
// columns at D = 64); measured slower there (its 152-register softmax
// warpgroups spill), so it is not selected.  One query tile per CTA with two
// CTAs per SM (two MMA lanes per SM) is supported too; at D = 64 it measured
// 6% slower windowed and no faster with the window off, so it is not selected.
template <int D>
struct PrefillShape {
  // query tiles per CTA = softmax warpgroups
  static constexpr int QT = 2;
  static constexpr int BN = 128;                      // keys per tile
  static constexpr int THREADS = (QT + 1) * 128;      // + producer, MMA issuer, 2 idle warps
  static constexpr int CTAS_PER_SM = (QT == 1) ? 2 : 1;
  // Registers: launched at 65536 / (THREADS x CTAS_PER_SM) per thread; the
  // softmax warpgroups grow and the last warpgroup shrinks to 56:
  //   QT = 2: 256 x 224 + 128 x 56 = 64512;  QT = 3: 384 x 152 + 128 x 56 = 65536;
  //   QT = 1 (two CTAs per SM): 2 x (128 x 200 + 128 x 56) = 65536.
  static constexpr uint32_t REGS_SOFTMAX = (QT == 3) ? 152 : (QT == 1) ? 200 : 224;
  static constexpr uint32_t REGS_OTHER = 56;
  static constexpr uint32_t TMEM_COLS = (QT == 1) ? 256 : 512;  // S tiles then O tiles
};

struct PrefillParams {
  uint16_t* out;      // [B, Nq, Hq, D] bf16
  float* lse;         // [B, Hq, Nq] or null
  int B, Nq, Nk, Hq, Hkv, G;
  int num_ctas_q;     // CTAs along the query axis (256 rows each)
  int qk_off;         // q_pos0 - k_pos0: query t is at relative position qk_off + t, key j at j
  float scale_log2;   // softmax scale * log2(e)
  int g8;             // 1: pairs share thresholds in groups of 8
  int T[64];          // per-pair thresholds (nondecreasing), clamped to INT32_MAX
  // block mask, or null: query tile qt (rows 128 qt ..) attends key tile kt
  // (keys 128 kt ..) iff bit kt % 32 of word kt / 32 of row (b, h, qt) is set;
  // rows of mask_words words, [B, Hq, ceil(Nq / 128), mask_words]
  const uint32_t* block_mask;
  int mask_words;
  // explicit positions (the POS kernel): query t of sequence b at
  // q_pos[b * q_pos_stride + t], key j at k_pos[b * k_pos_stride + j], both
  // non-decreasing along the sequence; k_pos rows 16-byte aligned and padded
  // to a multiple of 128 keys
  const int32_t* q_pos;
  const int32_t* k_pos;
  int64_t q_pos_stride, k_pos_stride;
  // Work items: the CTA of query block bx (longest rows first) of head h and
  // sequence b is item (b * Hq + h) * num_ctas_q + bx, its linear block index
  // in the unsplit grid.  The unsplit kernel runs items below item_end.
  int64_t item_end;
  // The split kernel runs items split_item0 .. split_item0 + split_items - 1,
  // each as kv_splits CTAs (block x = local item * kv_splits + s): part s
  // attends only key tiles [s * split_tiles, (s + 1) * split_tiles) and writes
  // its rows' result, normalised over that range's keys, to part_o
  // [kv_splits][split_items * 256][D] fp32 and the log2-sum-exp of its scores
  // (-inf when it has none) to part_l [kv_splits][split_items * 256], at row
  // (s * split_items + local item) * 256 + the row's index within the item.
  int split_item0, split_items;
  // unsplit grid (Hq, B, num_ctas_q) instead of (num_ctas_q, Hq, B): every head's
  // heaviest query blocks are dispatched before any head's lighter ones (g = 8 only)
  int heads_fast;
  int kv_splits, split_tiles;
  float* part_o;
  float* part_l;
};

template <int D>
struct PrefillSmem {
  static constexpr int QT = PrefillShape<D>::QT, BN = PrefillShape<D>::BN;
  static constexpr int NS = (D == 64 && QT > 1) ? 4 : 2;  // K/V ring depth
  static constexpr int QTILE = kBM * D * 2;          // one Q tile in bytes
  static constexpr int KTILE = BN * D * 2;           // one K or V tile in bytes
  static constexpr int PANEL_Q = kBM * 16;           // one 8-dim panel of a Q tile
  static constexpr int PANEL_K = BN * 16;            // one 8-dim panel of a K tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QT * QTILE;
  static constexpr int OFF_V = OFF_K + NS * KTILE;
  static constexpr int OFF_QM = OFF_V + NS * KTILE;          // masked first k-step of Q, per tile
  static constexpr int OFF_CT = OFF_QM + QT * 2 * PANEL_Q;    // per-warp transposed K pairs
  static constexpr int OFF_T = OFF_CT + 4 * QT * kCT * 32 * 4;  // thresholds (64 x int32)
  static constexpr int OFF_QR = OFF_T + 64 * 4;               // first / last query position per tile
  static constexpr int OFF_KP = OFF_QR + 16 * 4;              // key positions of each ring stage
  static constexpr int OFF_BAR = OFF_KP + NS * BN * 4;
  // barriers: q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS],
  //           s_full[QT], p_full[QT], o_final[QT], qm_init[QT]
  static constexpr int NBAR = 1 + 4 * NS + 4 * QT;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_TMEM + 16;
  static constexpr int ALLOC = BYTES;
};

__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// G8: pairs share thresholds in groups of 8 (a compile-time switch, so the
// two correction paths do not share a register allocation).  MASK: a block
// mask selects the key tiles (compile-time too, so that the plain causal walk
// keeps its registers).  POS: explicit, non-decreasing positions per token;
// every column range that the contiguous kernel derives from a distance is
// found by a binary search over the key tile's positions instead.  SPLIT: the
// key range is split into p.kv_splits parts (a compile-time switch too: the
// unsplit kernel keeps its registers).
template <int D, bool G8, bool MASK, bool POS, bool SPLIT>
__global__ void __launch_bounds__(PrefillShape<D>::THREADS, PrefillShape<D>::CTAS_PER_SM)
prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ PrefillParams p) {
  using L = PrefillSmem<D>;
  constexpr int NS = L::NS;
  constexpr int QT = PrefillShape<D>::QT;   // query tiles per CTA
  constexpr int BN = PrefillShape<D>::BN;   // keys per tile
  constexpr int P = D / 2;
  constexpr int KS = D / 16;          // k-steps of the QK contraction (8 pairs each)
  constexpr int PANEL_Q = L::PANEL_Q;
  constexpr int PANEL_K = L::PANEL_K;
  constexpr int W_PROD = 4 * QT;      // producer warp (after the softmax warpgroups)
  constexpr int W_MMA = 4 * QT + 1;   // MMA issuer warp
  constexpr uint32_t TMEM_O = QT * BN;  // S_t at t * BN, O_t at TMEM_O + t * D
  constexpr uint32_t FULL = 0xffffffffu;

  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + L::OFF_Q;
  const uint32_t sK = sbase + L::OFF_K;
  const uint32_t sV = sbase + L::OFF_V;
  const uint32_t bar = sbase + L::OFF_BAR;
  const uint32_t q_full = bar;
  auto k_full = [&](int s) { return bar + 8 * (1 + s); };
  auto k_empty = [&](int s) { return bar + 8 * (1 + NS + s); };
  auto v_full = [&](int s) { return bar + 8 * (1 + 2 * NS + s); };
  auto v_empty = [&](int s) { return bar + 8 * (1 + 3 * NS + s); };
  auto s_full = [&](int t) { return bar + 8 * (1 + 4 * NS + t); };
  auto p_full = [&](int t) { return bar + 8 * (1 + 4 * NS + QT + t); };
  auto o_final = [&](int t) { return bar + 8 * (1 + 4 * NS + 2 * QT + t); };
  auto qm_init = [&](int t) { return bar + 8 * (1 + 4 * NS + 3 * QT + t); };

  const uint32_t sQM = sbase + L::OFF_QM;
  int* sT = reinterpret_cast<int*>(smem + L::OFF_T);  // per-pair thresholds, read by every role
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);

  // the 128-byte-swizzled V tiles need a 1024-byte aligned shared window
  if (sbase & 1023u) {
    if (threadIdx.x == 0) record_status(2 /* WPATTN_EUNSUPPORTED */);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int cq, h, b, part = 0, local_item = 0;
  if constexpr (SPLIT) {
    local_item = static_cast<int>(blockIdx.x) / p.kv_splits;
    part = static_cast<int>(blockIdx.x) % p.kv_splits;
    const int item = p.split_item0 + local_item;
    const int hb = item / p.num_ctas_q;
    cq = p.num_ctas_q - 1 - (item % p.num_ctas_q);
    h = hb % p.Hq;
    b = hb / p.Hq;
  } else if (G8 && p.heads_fast) {
    cq = p.num_ctas_q - 1 - blockIdx.z;  // longest rows first, across all heads
    h = blockIdx.x;
    b = blockIdx.y;
  } else {
    if ((static_cast<int64_t>(blockIdx.z) * p.Hq + blockIdx.y) * p.num_ctas_q + blockIdx.x >= p.item_end)
      return;  // an item the split kernel runs
    cq = p.num_ctas_q - 1 - blockIdx.x;  // longest rows first
    h = blockIdx.y;
    b = blockIdx.z;
  }
  const int kvh = h / p.G;
  const int nkt = (p.Nk + BN - 1) / BN;
  // the key tiles this CTA may attend: all of them, or its part's range
  const int kt_lo = SPLIT ? part * p.split_tiles : 0;
  const int kt_hi = SPLIT ? min(kt_lo + p.split_tiles, nkt) - 1 : nkt - 1;

  // Positions.  Without POS query i sits at qk_off + i and key j at j
  // (relative to the first key); with POS they are read from the arrays.
  const int32_t* qp_row = nullptr;
  const int32_t* kp_row = nullptr;
  if constexpr (POS) {
    qp_row = p.q_pos + (size_t)b * p.q_pos_stride;
    kp_row = p.k_pos + (size_t)b * p.k_pos_stride;
  }
  const int* sQR = reinterpret_cast<const int*>(smem + L::OFF_QR);  // POS: [t] first, [QT + t] last
  auto k_first = [&](int kt) -> int {   // position of key tile kt's first key
    if constexpr (POS) return __ldg(kp_row + BN * kt);
    else return BN * kt;
  };
  auto k_last = [&](int kt) -> int {    // position of its last key (contiguous: as if full)
    if constexpr (POS) return __ldg(kp_row + min(BN * kt + BN - 1, p.Nk - 1));
    else return BN * kt + BN - 1;
  };
  auto q_first = [&](int t) -> int {    // position of query tile t's first row
    if constexpr (POS) return sQR[t];
    else return p.qk_off + (QT * cq + t) * kBM;
  };
  // key tiles of query tile t: positions <= its last row, iterated from kt_top down
  auto last_key_tile = [&](int t) -> int {
    const int row0 = (QT * cq + t) * kBM;
    if (row0 >= p.Nq || p.Nk <= 0) return -1;
    if constexpr (POS) {
      // last key tile whose first key is not after the tile's last row
      const int i_max = __ldg(qp_row + min(row0 + kBM - 1, p.Nq - 1));
      int lo = 0, hi = nkt - 1, found = -1;
      while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        if (k_first(mid) <= i_max) { found = mid; lo = mid + 1; } else { hi = mid - 1; }
      }
      return found;
    }
    const int i_max = p.qk_off + min(row0 + kBM - 1, p.Nq - 1);
    if (i_max < 0) return -1;
    return min(i_max / BN, nkt - 1);
  };
  int kt_last[QT];
#pragma unroll
  for (int t = 0; t < QT; ++t) kt_last[t] = SPLIT ? min(last_key_tile(t), kt_hi) : last_key_tile(t);
  // Key tiles query tile t attends: at most its causal limit lim, and with a
  // block mask only those whose bit is set.  Largest such tile <= kt, or -1.
  const int nqt = (p.Nq + kBM - 1) / kBM;
  auto attended_below = [&](int t, int kt, int lim) -> int {
    kt = min(kt, lim);
    if (kt < kt_lo) return -1;
    if constexpr (!MASK) return kt;
    const uint32_t* row =
        p.block_mask + ((size_t)(b * p.Hq + h) * nqt + (QT * cq + t)) * p.mask_words;
    while (kt >= kt_lo) {
      const uint32_t w = __ldg(row + (kt >> 5)) & (0xFFFFFFFFu >> (31 - (kt & 31)));
      if (w) {
        const int u = (kt & ~31) + 31 - __clz(w);
        return u >= kt_lo ? u : -1;
      }
      kt = (kt & ~31) - 1;
    }
    return -1;
  };
  // The CTA's K/V stream: the key tiles some of its query tiles attend, from the
  // top down.  Step j of the stream is key tile kt_j; bit t of *mem says whether
  // query tile t attends it.  Every role walks the same stream.
  auto stream_below = [&](int kt, uint32_t* mem) -> int {
    if constexpr (!MASK) {  // every tile up to the causal limit: the stream is a countdown
      int top = -1;
#pragma unroll
      for (int t = 0; t < QT; ++t) top = max(top, kt_last[t]);
      const int u = min(kt, top);
      uint32_t bits = 0;
#pragma unroll
      for (int t = 0; t < QT; ++t) bits |= (u >= kt_lo && u <= kt_last[t]) ? (1u << t) : 0u;
      *mem = bits;
      return u < kt_lo ? -1 : u;
    }
    int a[QT], u = -1;
#pragma unroll
    for (int t = 0; t < QT; ++t) { a[t] = attended_below(t, kt, kt_last[t]); u = max(u, a[t]); }
    uint32_t bits = 0;
#pragma unroll
    for (int t = 0; t < QT; ++t) bits |= (u >= 0 && a[t] == u) ? (1u << t) : 0u;
    *mem = bits;
    return u;
  };
  uint32_t mem_top;
  const int kt_top = stream_below(kt_hi, &mem_top);  // first step of the stream, -1 if none
  // the step after key tile kt (for the roles that do not need the bits)
  auto stream_next = [&](int kt) -> int {
    if constexpr (!MASK) return kt > kt_lo ? kt - 1 : -1;
    uint32_t unused;
    return stream_below(kt - 1, &unused);
  };
  // Smallest distance of query tile t in key tile kt (negative on the diagonal).
  // Going down the key tiles it grows by 128, so the first kept pair of the
  // tile (p_min of that distance) only moves forward: advance it in place.
  auto advance_plo_k = [&](int t, int klast, int& plo) {
    const int dlo = q_first(t) - klast;
    while (plo < P && sT[plo] < dlo) ++plo;
  };
  // (the contiguous forms are written out: routed through the position lambdas
  // the MMA lane's code came out 2% slower on the 32K Qwen-shaped prefill)
  auto advance_plo = [&](int t, int kt, int& plo) {
    if constexpr (!POS) {
      const int dlo = p.qk_off + (QT * cq + t) * kBM - (BN * kt + BN - 1);
      while (plo < P && sT[plo] < dlo) ++plo;
    } else {
      advance_plo_k(t, k_last(kt), plo);
    }
  };
  // Split pair of the tile: pairs plo .. ps-1 (kept somewhere in the tile) are
  // left out of the contraction and added back where they are kept; pairs
  // ps .. P-1 are contracted and subtracted where they are pruned.  Splitting
  // at the pair first kept 32 past the tile's centre distance keeps both
  // correction sets small (each element only pays for pairs whose threshold
  // lies between its distance and the centre).  Groups of 8 pairs share a
  // threshold, so for g = 8 the split falls on a group start.
  // The centre distance grows along the walk, so the first pair kept past it
  // (psr, carried by the caller) is advanced in place like plo.
  auto split_pair_k = [&](int t, int kfirst, int plo, int& psr) -> int {
    if (plo >= P) return plo;
    const int dc = max(q_first(t) - kfirst, 0);  // row 0 to key 0
    const int target = dc > 0x7FFFFFDF ? 0x7FFFFFFF : dc + 32;
    while (psr < P && sT[psr] < target) ++psr;
    return min(max(psr, plo), P - (G8 ? 8 : 1));
  };
  auto split_pair = [&](int t, int kt, int plo, int& psr) -> int {
    if constexpr (!POS) {
      if (plo >= P) return plo;
      const int dc = max(p.qk_off + (QT * cq + t) * kBM - BN * kt, 0);  // row 0 to key 0
      const int target = dc > 0x7FFFFFDF ? 0x7FFFFFFF : dc + 32;
      while (psr < P && sT[psr] < target) ++psr;
      return min(max(psr, plo), P - (G8 ? 8 : 1));
    } else {
      return split_pair_k(t, k_first(kt), plo, psr);
    }
  };
  // POS: number of the first nv keys of a ring stage whose position is below x
  // (the stage's positions are sorted)
  auto col_below = [&](const int* kps, int nv, int x) -> int {
    int lo = 0, hi = nv;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (kps[mid] < x) lo = mid + 1; else hi = mid;
    }
    return lo;
  };

  if (threadIdx.x < 64) sT[threadIdx.x] = p.T[threadIdx.x];
  if constexpr (POS) {
    if (threadIdx.x < 2 * QT) {
      const int t = threadIdx.x % QT;
      const int row0 = (QT * cq + t) * kBM;
      const int row = threadIdx.x < QT ? row0 : row0 + kBM - 1;
      reinterpret_cast<int*>(smem + L::OFF_QR)[threadIdx.x] =
          row0 < p.Nq ? __ldg(qp_row + min(row, p.Nq - 1)) : 0;
    }
  }
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1 + 4 * QT);  // MMA commit + every softmax warp (they read K for corrections)
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int t = 0; t < QT; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(p_full(t), 4);
      mbar_init(o_final(t), 1);
      mbar_init(qm_init(t), 4);

    }
    fence_barrier_init();
  }
  if (warp == W_MMA) {
    tmem_alloc(smem_u32(tmem_slot), PrefillShape<D>::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= W_PROD) {
  regs_decrease<PrefillShape<D>::REGS_OTHER>();
  if (warp == W_PROD) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && kt_top >= 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      // a query tile wholly past Nq is not loaded (its rows are never used)
      int nq_tiles = 0;
      for (int t = 0; t < QT; ++t) nq_tiles += ((QT * cq + t) * kBM < p.Nq) ? 1 : 0;
      mbar_arrive_expect_tx(q_full, nq_tiles * L::QTILE);
      for (int t = 0; t < nq_tiles; ++t)
        for (int c = 0; c < D / 8; ++c)
          tma_load_4d(sQ + t * L::QTILE + c * PANEL_Q, &tmQ, q_full, 8 * c, (QT * cq + t) * kBM, h, b);
      int nk_issued = 0, nv_issued = 0;  // K / V tiles whose copies were issued
      bool ok_prod = true;
      for (int j = 0, kt = kt_top; kt >= 0; ++j, kt = stream_next(kt)) {
        const int s = j % NS;
        const uint32_t ph = (j / NS) & 1;
        if (j >= NS && !mbar_wait(k_empty(s), ph ^ 1)) { ok_prod = false; break; }
        mbar_arrive_expect_tx(k_full(s), L::KTILE + (POS ? BN * 4 : 0));
        for (int c = 0; c < D / 8; ++c)
          tma_load_4d(sK + s * L::KTILE + c * PANEL_K, &tmK, k_full(s), 8 * c, BN * kt, kvh, b);
        if constexpr (POS)  // the tile's key positions travel with its keys
          bulk_load(sbase + L::OFF_KP + s * BN * 4, kp_row + BN * kt, BN * 4, k_full(s));
        nk_issued = j + 1;
        if (j >= NS && !mbar_wait(v_empty(s), ph ^ 1)) { ok_prod = false; break; }
        mbar_arrive_expect_tx(v_full(s), L::KTILE);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sV + s * L::KTILE + c * (BN * 128), &tmV, v_full(s), 64 * c, BN * kt, kvh, b);
        nv_issued = j + 1;
      }
      if (!ok_prod) {
        // A wait ran out: copies issued into the ring may still be landing in
        // shared memory.  Wait (bounded) for the fill of every stage's last
        // issued tile, and for Q, before this CTA can leave; a tile older than
        // a stage's last one completed before its stage was reused.
        (void)mbar_wait(q_full, 0);
        for (int j = max(0, nk_issued - NS); j < nk_issued; ++j)
          (void)mbar_wait(k_full(j % NS), (j / NS) & 1);
        for (int j = max(0, nv_issued - NS); j < nv_issued; ++j)
          (void)mbar_wait(v_full(j % NS), (j / NS) & 1);
      }
    }
  } else if (warp == W_MMA) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && kt_top >= 0) {
      constexpr uint32_t idesc_qk = make_idesc_bf16(kBM, BN, 0, 0);
      constexpr uint32_t idesc_pv = make_idesc_bf16(kBM, D, 0, 1);
      bool ok = mbar_wait(q_full, 0);
      // per query tile (indices are compile-time after unrolling): PVs issued,
      // masked-Q barrier seen, planner state
      int cnt[QT], plo[QT], psr[QT];
      bool qm_seen[QT];
#pragma unroll
      for (int t = 0; t < QT; ++t) { cnt[t] = 0; plo[t] = 0; psr[t] = 0; qm_seen[t] = false; }
      // descriptors: start addresses advance by adding (byte offset >> 4);
      // LBO = D/16 panels: first half -> second half of a pair
      const uint64_t qdesc0 = make_sdesc(sQ, (D / 16) * PANEL_Q, 128, 0);
      const uint64_t qmdesc0 = make_sdesc(sQM, PANEL_Q, 128, 0);
      const uint64_t kdesc0 = make_sdesc(sK, (D / 16) * PANEL_K, 128, 0);
      const uint64_t vdesc0 = make_sdesc(sV, BN * 128, 1024, 2);
      // split pair of QK_t on key tile kt (in ring stage stage, already filled):
      // planned ahead of the wait for P_t
      auto plan_qk = [&](int t, int kt, int stage) -> int {
        if constexpr (POS) {
          const int* kps = reinterpret_cast<const int*>(smem + L::OFF_KP) + stage * BN;
          advance_plo_k(t, kps[min(BN, p.Nk - BN * kt) - 1], plo[t]);
          return split_pair_k(t, kps[0], plo[t], psr[t]);
        }
        advance_plo(t, kt, plo[t]);
        return split_pair(t, kt, plo[t], psr[t]);
      };
      auto issue_qk = [&](int t, int j, int ps) -> bool {
        if (!qm_seen[t]) {  // the softmax warps prepared the masked k-step of tile t's first tile
          if (!mbar_wait(qm_init(t), 0)) return false;
          qm_seen[t] = true;
        }
        const int k0 = ps >> 3;
        const uint64_t kbase = kdesc0 + (uint64_t)(((j % NS) * L::KTILE) >> 4);
        const uint64_t qbase = qdesc0 + (uint64_t)((t * L::QTILE) >> 4);
        const uint32_t d_tmem = tmem + t * BN;
        for (int ks = k0; ks < KS; ++ks) {
          // pairs 8*k0 .. ps-1 are not contracted: the first step reads a
          // copy of Q with those pairs zeroed
          const uint64_t ad = (ks == k0 && (ps & 7))
                                  ? qmdesc0 + (uint64_t)((t * 2 * PANEL_Q) >> 4)
                                  : qbase + (uint64_t)((ks * PANEL_Q) >> 4);
          umma_ss(d_tmem, ad, kbase + (uint64_t)((ks * PANEL_K) >> 4), idesc_qk, ks > k0 ? 1u : 0u);
        }
        umma_commit(s_full(t));
        return true;
      };
      if (ok && mbar_wait(k_full(0), 0)) {
        tc_fence_after();
#pragma unroll
        for (int t = 0; t < QT; ++t)
          if (ok && (MASK ? ((mem_top >> t) & 1u) != 0 : kt_last[t] >= kt_top) &&
              !issue_qk(t, 0, plan_qk(t, kt_top, 0)))
            ok = false;
        umma_commit(k_empty(0));
      } else {
        ok = false;
      }
      // without a mask, query tile t attends step kt iff kt <= kt_last[t] (no bits carried)
      uint32_t mem = MASK ? mem_top : 0u;
      for (int j = 0, kt = kt_top; ok && kt >= 0; ++j) {
        uint32_t mem_n = 0;
        int kt_n;
        if constexpr (MASK) kt_n = stream_below(kt - 1, &mem_n);
        else kt_n = kt > kt_lo ? kt - 1 : -1;
        const bool next = kt_n >= 0;
        if (next && !mbar_wait(k_full((j + 1) % NS), ((j + 1) / NS) & 1)) { ok = false; break; }
        if (!mbar_wait(v_full(j % NS), (j / NS) & 1)) { ok = false; break; }
        const uint64_t vbase = vdesc0 + (uint64_t)(((j % NS) * L::KTILE) >> 4);
#pragma unroll
        for (int t = 0; t < QT; ++t) {
          const bool in_n = MASK ? ((mem_n >> t) & 1u) != 0 : kt_n <= kt_last[t];
          const bool in_j = MASK ? ((mem >> t) & 1u) != 0 : kt <= kt_last[t];
          const bool do_qk = ok && next && in_n;
          const int ps_n = do_qk ? plan_qk(t, kt_n, (j + 1) % NS) : 0;
          if (ok && in_j) {
            if (!mbar_wait_handoff(p_full(t), cnt[t] & 1)) { ok = false; }
            if (ok) {
              tc_fence_after();
#pragma unroll
              for (int ks = 0; ks < BN / 16; ++ks)
                umma_ts(tmem + TMEM_O + t * D, tmem + t * BN + ks * 8,
                        vbase + (uint64_t)((ks * 2048) >> 4), idesc_pv, (cnt[t] > 0 || ks > 0) ? 1u : 0u);
              ++cnt[t];
            }
          }
          if (ok && do_qk && !issue_qk(t, j + 1, ps_n)) ok = false;
        }
        if (!ok) break;
        umma_commit(v_empty(j % NS));
        if (next) umma_commit(k_empty((j + 1) % NS));
        kt = kt_n;
        if constexpr (MASK) mem = mem_n;
      }
      // O_t final: every MMA issued so far has completed once this arrives
      for (int t = 0; t < QT; ++t) umma_commit(o_final(t));
      if (!ok) mbar_wait(o_final(0), 0);
    }
  }
  } else {
    regs_increase<PrefillShape<D>::REGS_SOFTMAX>();
    // ------------------------------------------------------------- softmax
    const int t = warp >> 2;                   // query tile of this warpgroup
    const int wq = warp & 3;                   // TMEM lane quarter
    const int r = wq * 32 + lane;              // row within the tile = TMEM lane
    const int row = (QT * cq + t) * kBM + r;   // query index
    // position of this row (relative to the first key without POS)
    const int i_pos = POS ? __ldg(qp_row + min(row, p.Nq - 1)) : p.qk_off + row;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t tS = lane_base + t * BN;
    const uint32_t tO = lane_base + TMEM_O + t * D;
    const uint8_t* smem_q = smem + L::OFF_Q + t * L::QTILE;
    uint8_t* smem_qm = smem + L::OFF_QM + t * 2 * PANEL_Q;
    const int i_tile0 = q_first(t);           // position of the tile's first row
    const int my_kt_last = SPLIT ? min(last_key_tile(t), kt_hi) : last_key_tile(t);
    int my_next = attended_below(t, my_kt_last, my_kt_last);  // this tile's next key tile, -1 when done
    float m_ref = -INFINITY;   // exponent reference of O and l (log2 units)
    float l_run = 0.f;
    int cnt = 0;
    bool ok = true;

    // Copy of Q's first contracted k-step for a key tile whose split pair is
    // ps, with the pairs below ps zeroed (the MMA reads it instead of Q).
    // (g = 1) the split pair whose masked copy the buffer holds: the split pair only
    // moves forward along the walk, and far from the diagonal it stays put for dozens
    // of key tiles, so the copy and its proxy fence are skipped while it does
    int qm_ps = -1;
    auto write_masked_q = [&](int ps) {
      const int rz = ps & 7;
      if (rz == 0 || (ps >> 3) >= KS) return;
      if constexpr (!G8) {
        if (ps == qm_ps) return;
        qm_ps = ps;
      }
      uint4 lo = *reinterpret_cast<const uint4*>(smem_q + (ps >> 3) * PANEL_Q + r * 16);
      uint4 hi = *reinterpret_cast<const uint4*>(smem_q + (P / 8 + (ps >> 3)) * PANEL_Q + r * 16);
      const uint32_t m0 = (rz > 0 ? 0u : 0xFFFFu) | (rz > 1 ? 0u : 0xFFFF0000u);
      const uint32_t m1 = (rz > 2 ? 0u : 0xFFFFu) | (rz > 3 ? 0u : 0xFFFF0000u);
      const uint32_t m2 = (rz > 4 ? 0u : 0xFFFFu) | (rz > 5 ? 0u : 0xFFFF0000u);
      const uint32_t m3 = (rz > 6 ? 0u : 0xFFFFu) | 0xFFFF0000u;
      lo.x &= m0; lo.y &= m1; lo.z &= m2; lo.w &= m3;
      hi.x &= m0; hi.y &= m1; hi.z &= m2; hi.w &= m3;
      *reinterpret_cast<uint4*>(smem_qm + r * 16) = lo;
      *reinterpret_cast<uint4*>(smem_qm + PANEL_Q + r * 16) = hi;
      fence_proxy_async_smem();
    };

    // Q is read from shared memory for the masked copy and the corrections
    // (it is loaded only when the CTA's stream has a key tile)
    ok = kt_top < 0 || __all_sync(FULL, mbar_wait(q_full, 0));
    int plo_next = 0;
    if (my_next >= 0) advance_plo(t, my_next, plo_next); else plo_next = P;
    int psr = 0;
    int ps_next = my_next >= 0 ? split_pair(t, my_next, plo_next, psr) : P;
    if (ok && my_next >= 0) write_masked_q(ps_next);
    __syncwarp();
    if (lane == 0) mbar_arrive(qm_init(t));

    for (int j = 0, kt = kt_top; ok && kt >= 0; ++j, kt = stream_next(kt)) {
      const int s = j % NS;
      if (MASK ? kt != my_next : kt > my_kt_last) {
        // a key tile this query tile does not attend (past its rows, or
        // masked out): only release K.  Wait for the stage's fill first, so
        // that this arrival counts towards step j and not towards an earlier
        // phase of the same stage.
        if (!__all_sync(FULL, mbar_wait(k_full(s), (j / NS) & 1))) { ok = false; break; }
        __syncwarp();
        if (lane == 0) mbar_arrive(k_empty(s));
        continue;
      }
      const int kp0 = BN * kt;
      // POS: the stage's key positions (the first nv are keys), read after its fill;
      // this row attends columns [0, c_caus)
      const int* kps = reinterpret_cast<const int*>(smem + L::OFF_KP) + s * BN;
      int nv = BN, k_lo = 0, k_hi = 0, c_caus = 0;
      if constexpr (POS) {
        if (!__all_sync(FULL, mbar_wait(k_full(s), (j / NS) & 1))) { ok = false; break; }
        nv = min(BN, p.Nk - kp0);
        k_lo = kps[0];
        k_hi = kps[nv - 1];
        // rows at or past the tile's last key attend all of it (no search)
        c_caus = i_pos >= k_hi ? nv : col_below(kps, nv, i_pos + 1);
      }
      const int d_row = i_pos - (POS ? k_lo : kp0);  // distance to the tile's first key
      const int plo = plo_next, ps = ps_next;
      const bool all_pruned = plo >= P;
      if constexpr (MASK) my_next = attended_below(t, kt - 1, my_kt_last);
      else my_next = kt > kt_lo ? kt - 1 : -1;  // below the first attended tile, every tile is attended
      if (my_next >= 0) {
        advance_plo(t, my_next, plo_next);
        ps_next = split_pair(t, my_next, plo_next, psr);
      }

      // Per-element corrections, d = d_row - c for column c of the tile:
      //   pairs plo .. ps-1 were left out of the contraction: add their terms
      //   where they are kept (0 <= d <= T);
      //   pairs ps .. P-1 were contracted: subtract their terms where they
      //   are pruned (d > T).  Thresholds grow with the pair index.
      // For g = 1 they depend on Q and K only, so they are summed into sc
      // while the tensor core is still computing S, and S is added once it
      // is ready; for g = 8 they are applied to S in TMEM before it is read.
      const bool need_sub = !all_pruned && __any_sync(FULL, d_row > sT[ps]);
      const int d_last = POS ? i_pos - k_hi : d_row - (BN - 1);  // distance to the last key
      const bool need_add = !all_pruned && ps > plo &&
                            __any_sync(FULL, d_row >= 0 && d_last <= sT[ps - 1]);
      const bool corr = need_sub || need_add;
      // K stage s is released below; waiting for its fill first makes the
      // arrival count towards iteration j (the stage's previous phase is over)
      if constexpr (!POS) {
        if (!__all_sync(FULL, mbar_wait(k_full(s), (j / NS) & 1))) { ok = false; break; }
      }
      float sc[BN];
      if (!corr) {  // K stage s is no longer read by this warp
        __syncwarp();
        if (lane == 0) mbar_arrive(k_empty(s));
      }

      if (!__all_sync(FULL, mbar_wait_handoff(s_full(t), cnt & 1))) { ok = false; break; }
      tc_fence_after();
      if (corr && G8) {
        const uint8_t* kb = smem + L::OFF_K + s * L::KTILE;
        // whole groups of 8 pairs share a threshold: one 16-dim dot product per element
#pragma unroll 1
        for (int gp = plo; gp < P; gp += 8) {
          const bool sub = gp >= ps;
          const int T = sT[gp];
          int c_lo, c_hi;  // columns of this row that take the group's term
          if constexpr (POS) {
            const int cth = col_below(kps, nv, i_pos - T);  // columns farther than T
            c_lo = sub ? 0 : cth;
            c_hi = sub ? cth - 1 : c_caus - 1;
          } else if (sub) {
            c_lo = 0;
            c_hi = d_row > T ? min(d_row - T - 1, BN - 1) : -1;
          } else {
            c_lo = T >= d_row ? 0 : d_row - T;
            c_hi = min(d_row, BN - 1);
          }
          if (!__any_sync(FULL, c_lo <= c_hi)) {
            if (sub) break;  // later groups are pruned at even fewer columns
            continue;
          }
          const float sgn = sub ? -1.f : 1.f;
          const int grp = gp >> 3;
          // The group's 16-dim products for this warp's 32 rows on the tensor
          // cores (mma.sync m16n8k16): A = Q rows (dims 8 grp.. then P + 8 grp..),
          // B = K rows of the chunk's keys.  Lane (gid, tig) gets rows gid (+8)
          // and keys 2 tig (+1) of each 16 x 8 block; a per-warp scratch turns
          // them into one row per lane.  A: matrix m of the ldmatrix = rows
          // 8 (m & 1) .., first (m < 2) or second half of the group.
          const int qm = lane >> 3, qi = lane & 7;
          uint32_t afr[2][4];
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            const int row_a = wq * 32 + 16 * mt + 8 * (qm & 1) + qi;
            const int pan_a = (qm >> 1) ? P / 8 + grp : grp;
            ldsm_x4(smem_u32(smem_q) + pan_a * PANEL_Q + row_a * 16, afr[mt][0], afr[mt][1],
                    afr[mt][2], afr[mt][3]);
          }
          float* scr = reinterpret_cast<float*>(smem + L::OFF_CT) + warp * (32 * 16);  // [32 rows][16 keys]
#pragma unroll 1
          for (int cc = 0; cc < BN / 32; ++cc) {
            const int lo = c_lo - 32 * cc, hi = c_hi - 32 * cc;  // chunk-local range
            if (!__any_sync(FULL, lo <= 31 && hi >= 0 && lo <= hi)) continue;
            float v[32];
            tmem_ld32(tS + 32 * cc, v);
            tmem_ld_wait();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              // B: matrix m = keys 8 (m >> 1) .., first (m even) or second half of the group
              const int key = 32 * cc + 16 * half + 8 * (qm >> 1) + qi;
              const int pan_b = (qm & 1) ? P / 8 + grp : grp;
              uint32_t b00, b01, b10, b11;
              ldsm_x4(smem_u32(kb) + pan_b * PANEL_K + key * 16, b00, b01, b10, b11);
              float acc[2][2][4];
#pragma unroll
              for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                  for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
#pragma unroll
              for (int mt = 0; mt < 2; ++mt) {
                mma_16816_bf16(acc[mt][0], afr[mt][0], afr[mt][1], afr[mt][2], afr[mt][3], b00, b01);
                mma_16816_bf16(acc[mt][1], afr[mt][0], afr[mt][1], afr[mt][2], afr[mt][3], b10, b11);
              }
              __syncwarp();                 // the previous half's rows have been read
#pragma unroll
              for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                  const int rr = 16 * mt + (lane >> 2), cl = 8 * nt + 2 * (lane & 3);
                  *reinterpret_cast<float2*>(scr + rr * 16 + cl) = make_float2(acc[mt][nt][0], acc[mt][nt][1]);
                  *reinterpret_cast<float2*>(scr + (rr + 8) * 16 + cl) = make_float2(acc[mt][nt][2], acc[mt][nt][3]);
                }
              __syncwarp();
              const float4* mine = reinterpret_cast<const float4*>(scr + lane * 16);
#pragma unroll
              for (int c4 = 0; c4 < 4; ++c4) {
                const float4 x = mine[c4];
                const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int c = 16 * half + 4 * c4 + e;
                  if (c >= lo && c <= hi) v[c] = fmaf(sgn, xs[e], v[c]);
                }
              }
            }
            tmem_st32(tS + 32 * cc, v);
          }
        }
        tmem_st_wait();
        __syncwarp();
        if (lane == 0) mbar_arrive(k_empty(s));
      }
      if (corr && !G8) {
        // One pair per term, applied to S in TMEM like the groups above, its
        // products on the tensor cores: per 32-column chunk, the pairs whose
        // thresholds fall inside the block's distances; a pair's product is
        // its group's MMA with every A element but the pair's two dims zeroed.
        const uint8_t* kb = smem + L::OFF_K + s * L::KTILE;
        float* scr = reinterpret_cast<float*>(smem + L::OFF_CT) + warp * (32 * 16);  // [32 rows][16 keys]
        const int qm = lane >> 3, qi = lane & 7;
        const int T_lo = ps > plo ? sT[ps - 1] : 0;
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          if (POS && 32 * cc >= nv) break;                 // no key in this chunk
          // distance at the chunk's first column
          const int dc = POS ? i_pos - kps[32 * cc] : d_row - 32 * cc;
          const int dmax = __shfl_sync(FULL, dc, 31);      // largest distance of the block
          const int dmin = POS ? max(__shfl_sync(FULL, i_pos - kps[min(32 * cc + 31, nv - 1)], 0), 0)
                               : max(__shfl_sync(FULL, dc, 0) - 31, 0);
          if (dmax < 0) continue;                          // wholly acausal
          // pairs ps .. pb-1 are pruned somewhere in the block, pa .. ps-1 kept somewhere
          int pb = ps;
          if (need_sub)
            while (pb < P && sT[pb] < dmax) ++pb;
          int pa = ps;
          if (need_add && T_lo >= dmin)
            while (pa > plo && sT[pa - 1] >= dmin) --pa;
          if (pa >= pb) continue;
          float v[32];
          tmem_ld32(tS + 32 * cc, v);
          tmem_ld_wait();
          uint32_t afr[2][4];
          int cur = -1;
#pragma unroll 1
          for (int pp = pa; pp < pb; ++pp) {
            const int grp = pp >> 3;
            if (grp != cur) {  // A: this warp's Q rows of the group (matrix m: rows 8 (m & 1) .., half m >> 1)
              cur = grp;
#pragma unroll
              for (int mt = 0; mt < 2; ++mt) {
                const int row_a = wq * 32 + 16 * mt + 8 * (qm & 1) + qi;
                const int pan_a = (qm >> 1) ? P / 8 + grp : grp;
                ldsm_x4(smem_u32(smem_q) + pan_a * PANEL_Q + row_a * 16, afr[mt][0], afr[mt][1],
                        afr[mt][2], afr[mt][3]);
              }
            }
            const int T = sT[pp];
            int lo, hi;  // chunk columns of this row that take the pair's term
            float sgn;
            if constexpr (POS) {
              // chunk columns before cth are farther than T
              const int cth = col_below(kps, nv, i_pos - T) - 32 * cc;
              if (pp >= ps) {
                lo = 0;
                hi = min(cth, 32) - 1;
                sgn = -1.f;
              } else {
                lo = max(cth, 0);
                hi = min(c_caus - 32 * cc, 32) - 1;
                sgn = 1.f;
              }
            } else if (pp >= ps) {
              lo = 0;
              hi = dc > T ? min(dc - T, 32) - 1 : -1;
              sgn = -1.f;
            } else {
              lo = T >= dc ? 0 : dc - T;
              hi = min(dc, 31);
              sgn = 1.f;
            }
            if (!__any_sync(FULL, lo <= hi)) continue;
            // keep only the pair's dims: A register halves hold pairs 8 grp + 2 tig (+1)
            const int jp = pp & 7;
            const uint32_t keep = ((lane & 3) == (jp >> 1)) ? ((jp & 1) ? 0xFFFF0000u : 0x0000FFFFu) : 0u;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              // B: matrix m = keys 8 (m >> 1) .., first (m even) or second half of the group
              const int key = 32 * cc + 16 * half + 8 * (qm >> 1) + qi;
              const int pan_b = (qm & 1) ? P / 8 + grp : grp;
              uint32_t b00, b01, b10, b11;
              ldsm_x4(smem_u32(kb) + pan_b * PANEL_K + key * 16, b00, b01, b10, b11);
              float acc[2][2][4];
#pragma unroll
              for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                  for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
#pragma unroll
              for (int mt = 0; mt < 2; ++mt) {
                const uint32_t a0 = afr[mt][0] & keep, a1 = afr[mt][1] & keep;
                const uint32_t a2 = afr[mt][2] & keep, a3 = afr[mt][3] & keep;
                mma_16816_bf16(acc[mt][0], a0, a1, a2, a3, b00, b01);
                mma_16816_bf16(acc[mt][1], a0, a1, a2, a3, b10, b11);
              }
              __syncwarp();                 // the scratch's previous rows have been read
#pragma unroll
              for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                  const int rr = 16 * mt + (lane >> 2), cl = 8 * nt + 2 * (lane & 3);
                  *reinterpret_cast<float2*>(scr + rr * 16 + cl) = make_float2(acc[mt][nt][0], acc[mt][nt][1]);
                  *reinterpret_cast<float2*>(scr + (rr + 8) * 16 + cl) = make_float2(acc[mt][nt][2], acc[mt][nt][3]);
                }
              __syncwarp();
              const float4* mine = reinterpret_cast<const float4*>(scr + lane * 16);
#pragma unroll
              for (int c4 = 0; c4 < 4; ++c4) {
                const float4 x = mine[c4];
                const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int c = 16 * half + 4 * c4 + e;
                  if (c >= lo && c <= hi) v[c] = fmaf(sgn, xs[e], v[c]);
                }
              }
            }
          }
          tmem_st32(tS + 32 * cc, v);
        }
        tmem_st_wait();
        __syncwarp();
        if (lane == 0) mbar_arrive(k_empty(s));
      }
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) tmem_ld32(tS + 32 * cc, &sc[32 * cc]);
      tmem_ld_wait();
      // the loaded values are only defined after the wait: keep every use of
      // them below it (an empty asm that takes each register as an operand)
#pragma unroll
      for (int c = 0; c < BN; ++c) asm volatile("" : "+f"(sc[c]));

      if (all_pruned) {
#pragma unroll
        for (int c = 0; c < BN; ++c) sc[c] = 0.f;   // every pair pruned: score 0
      }

      // causal mask (d < 0) and the ragged key tail: columns c > cm
      const bool need_mask = POS ? (i_tile0 - k_hi < 0) || (nv < BN)
                                 : (i_tile0 - (kp0 + BN - 1) < 0) || (kp0 + BN > p.Nk);
      int cm = BN - 1;
      if (need_mask) {
        // last column with d >= 0, and the last real key
        cm = POS ? c_caus - 1 : min(max(min(d_row, p.Nk - 1 - kp0), -1), BN);
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c > cm) sc[c] = -INFINITY;
      }

      // Row max first, then the exponentials against the (lazily moved) reference.
      const float sl = p.scale_log2;
      auto tile_max = [&]() -> float {
        if constexpr (BN == 96) {
          float a12[12];
#pragma unroll
          for (int k = 0; k < 12; ++k)
            a12[k] = max3(max3(sc[8 * k], sc[8 * k + 1], sc[8 * k + 2]),
                          max3(sc[8 * k + 3], sc[8 * k + 4], sc[8 * k + 5]),
                          fmaxf(sc[8 * k + 6], sc[8 * k + 7]));
          const float b0 = max3(a12[0], a12[1], a12[2]), b1 = max3(a12[3], a12[4], a12[5]);
          const float b2 = max3(a12[6], a12[7], a12[8]), b3 = max3(a12[9], a12[10], a12[11]);
          return fmaxf(max3(b0, b1, b2), b3) * sl;
        }
        float a16[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          a16[k] = max3(max3(sc[8 * k], sc[8 * k + 1], sc[8 * k + 2]),
                        max3(sc[8 * k + 3], sc[8 * k + 4], sc[8 * k + 5]),
                        fmaxf(sc[8 * k + 6], sc[8 * k + 7]));
        float b6[6];
#pragma unroll
        for (int k = 0; k < 5; ++k) b6[k] = max3(a16[3 * k], a16[3 * k + 1], a16[3 * k + 2]);
        b6[5] = a16[15];
        return max3(max3(b6[0], b6[1], b6[2]), max3(b6[3], b6[4], b6[5]), -INFINITY) * sl;
      };
      // p for every column against reference m, packed to bf16 pairs in pk;
      // returns the row sum of p.  With 96-key tiles P is stored 16 columns
      // at a time as it is produced (fewer live registers).
      uint32_t pk[BN / 2];
      auto exps = [&](float m) -> float {
        const float nm = (m == -INFINITY) ? 0.f : -m;
        float acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.f;
#pragma unroll
        for (int i = 0; i < BN / 2; ++i) {
          const int c = 2 * i;
          float x0, x1, e0, e1;
          fma2(x0, x1, sc[c], sc[c + 1], sl, sl, nm, nm);
          e0 = ex2_approx(x0);
          e1 = ex2_approx(x1);
          add2(acc[2 * (i & 3)], acc[2 * (i & 3) + 1], acc[2 * (i & 3)], acc[2 * (i & 3) + 1], e0, e1);
          pk[i] = pack_bf16x2(e0, e1);
          if constexpr (BN == 96) {
            if ((i & 15) == 15) tmem_st16u(tS + (i - 15), &pk[i - 15]);
          }
        }
        return ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
      };

      const float mt = tile_max();
      // lazy rescale: move the reference only when the max grew by > 8 (x256).
      // s_full of this tile implies the previous PV of this tile has completed.
      float f = 1.f;
      if (cnt == 0) {
        m_ref = mt;
      } else if (mt > m_ref + 8.f) {
        f = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - mt);
        m_ref = mt;
      }
      if (cnt > 0 && __any_sync(FULL, f != 1.f)) {
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          float o[32];
          tmem_ld32(tO + 32 * cc, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= f;
          tmem_st32(tO + 32 * cc, o);
        }
      }
      const float rowsum = exps(m_ref);
      l_run = l_run * f + rowsum;
      if constexpr (BN == 128) {     // P overwrites the first 64 columns of S
        tmem_st32u(tS, &pk[0]);
        tmem_st32u(tS + 32, &pk[32]);
      }
      // the next tile's masked Q step, before P is released to the MMA warp
      if (MASK ? my_next >= 0 : kt > kt_lo) write_masked_q(ps_next);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full(t));
      ++cnt;
    }

    // epilogue: O / l
    const bool row_ok = row < p.Nq;
    const size_t out_row = ((size_t)b * p.Nq + (row_ok ? row : 0)) * p.Hq + h;
    uint16_t* orow = p.out + out_row * D;
    if (cnt > 0) {
      ok = __all_sync(FULL, mbar_wait(o_final(t), 0)) && ok;
      tc_fence_after();
    }
    const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
    // a split's part: fp32 O / l over its keys and the log2-sum-exp of its scores
    const size_t part_row =
        SPLIT ? ((size_t)part * p.split_items + local_item) * (QT * kBM) + t * kBM + r : 0;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      float o[32];
      if (cnt > 0) {
        tmem_ld32(tO + 32 * cc, o);
        tmem_ld_wait();
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = (cnt > 0) ? o[e] * inv : 0.f;
      if constexpr (SPLIT) {
        if (row_ok) {
          float4* prow = reinterpret_cast<float4*>(p.part_o + part_row * D + 32 * cc);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            prow[v4] = make_float4(o[4 * v4], o[4 * v4 + 1], o[4 * v4 + 2], o[4 * v4 + 3]);
        }
        continue;
      }
      if (row_ok) {
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          uint4 w;
          w.x = pack_bf16x2(o[8 * v4 + 0], o[8 * v4 + 1]);
          w.y = pack_bf16x2(o[8 * v4 + 2], o[8 * v4 + 3]);
          w.z = pack_bf16x2(o[8 * v4 + 4], o[8 * v4 + 5]);
          w.w = pack_bf16x2(o[8 * v4 + 6], o[8 * v4 + 7]);
          *reinterpret_cast<uint4*>(orow + 32 * cc + 8 * v4) = w;
        }
      }
    }
    if (SPLIT && row_ok)
      p.part_l[part_row] = (cnt > 0 && l_run > 0.f) ? m_ref + __log2f(l_run) : -INFINITY;
    else if (row_ok && p.lse)
      p.lse[((size_t)b * p.Hq + h) * p.Nq + row] =
          (l_run > 0.f) ? (m_ref + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == W_MMA) tmem_dealloc(tmem, PrefillShape<D>::TMEM_COLS);
}

// Byte block mask [rows, nkb] (nonzero = attended) -> the kernel's bit rows of
// mask_words words: bit kb % 32 of word kb / 32, zero past nkb.  One thread
// per word.
__global__ void __launch_bounds__(256)
pack_block_mask_kernel(const uint8_t* __restrict__ mask, uint32_t* __restrict__ words, int64_t rows,
                       int nkb, int mask_words) {
  const uint64_t idx = static_cast<uint64_t>(blockIdx.x) * 256u + threadIdx.x;
  if (idx >= static_cast<uint64_t>(rows) * static_cast<uint64_t>(mask_words)) return;
  const uint64_t r = idx / static_cast<uint64_t>(mask_words);
  const int wi = static_cast<int>(idx % static_cast<uint64_t>(mask_words));
  const uint8_t* src = mask + r * static_cast<uint64_t>(nkb);
  uint32_t w = 0;
  for (int i = 0; i < 32; ++i) {
    const int kb = wi * 32 + i;
    if (kb < nkb && src[kb]) w |= 1u << i;
  }
  words[idx] = w;
}

// Merge of the parts of the split kernel's items (one block per row of an
// item, one thread per head dim): with w_s = 2^(l_s - max l), out = sum_s
// w_s o_s / sum_s w_s and lse = ln 2 * (max l + log2 sum_s w_s); a row none
// of whose parts has a key gets 0 and -inf.
template <int D>
__global__ void __launch_bounds__(D)
prefill_combine_kernel(const __grid_constant__ PrefillParams p) {
  constexpr int ROWS = PrefillShape<D>::QT * kBM;   // query rows of an item
  const int local_item = static_cast<int>(blockIdx.x) / ROWS;
  const int lr = static_cast<int>(blockIdx.x) % ROWS;
  const int item = p.split_item0 + local_item;
  const int hb = item / p.num_ctas_q;
  const int cq = p.num_ctas_q - 1 - (item % p.num_ctas_q);
  const int h = hb % p.Hq, b = hb / p.Hq;
  const int t = cq * ROWS + lr;
  if (t >= p.Nq) return;
  const int e = threadIdx.x;
  const size_t prow = (size_t)local_item * ROWS + lr;
  const size_t pstride = (size_t)p.split_items * ROWS;   // rows of one part
  float M = -INFINITY;
  for (int s = 0; s < p.kv_splits; ++s) M = fmaxf(M, p.part_l[s * pstride + prow]);
  float W = 0.f, acc = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < p.kv_splits; ++s) {
      const float ls = p.part_l[s * pstride + prow];
      const float w = ls == -INFINITY ? 0.f : ex2_approx(ls - M);
      W += w;
      acc = fmaf(w, p.part_o[(s * pstride + prow) * D + e], acc);
    }
  }
  const float val = W > 0.f ? acc / W : 0.f;
  p.out[(((size_t)b * p.Nq + t) * p.Hq + h) * D + e] = static_cast<uint16_t>(pack_bf16x2(val, 0.f) & 0xFFFFu);
  if (p.lse && e == 0)
    p.lse[((size_t)b * p.Hq + h) * p.Nq + t] =
        W > 0.f ? (M + __log2f(W)) * 0.69314718055994530942f : -INFINITY;
}

}  // namespace wpattn
