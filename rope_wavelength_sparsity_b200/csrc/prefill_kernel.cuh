// Windowed causal attention prefill for sm_100a (TMA + tcgen05 + TMEM).
//
// "ATFlash: Per-RoPE-Wavelength Attention Windows", Abstract: the window is a
// slice of the query-key contraction axis and the online-softmax recurrence
// is left untouched.  "WavePrune", Original abstract and summary: head dims
// are grouped in blocks of 16 so the pruned contraction still runs on the
// Tensor Cores.
//
// One CTA owns 128 query rows of one (batch, query head) and walks the key
// tiles from the diagonal outwards.  Warp roles:
//   warps 0-3  softmax: row r of the tile is TMEM lane r; they read S from
//              TMEM, subtract the pairs that are pruned at some but not all
//              of the tile's distances, mask, run the online softmax with a
//              lazily rescaled O, write P (bf16) to shared memory and finish
//              with O / l.
//   warp 4     TMA producer: Q once, then K and V tiles into a ring.
//   warp 5     MMA issuer (one lane): S = Q K^T over the active k-steps, then
//              O += P V; owns the TMEM allocation.
//
// Shared-memory layouts.  Q and K use the no-swizzle canonical K-major layout
// with one 16-byte column panel per 8 head dims: panel c holds dims
// [8c, 8c+8) of all 128 rows (row r at byte 16 r), panels are 2 KB apart.
// A K=16 MMA step reads two core-matrix columns that are LBO bytes apart, so
// with LBO = (D/16) * 2 KB the step m pairs panel m (dims 8m..8m+7, the first
// halves of pairs 8m..8m+7) with panel D/16 + m (their second halves): every
// k-step carries 8 whole RoPE pairs, and skipping steps below k0 drops exactly
// the pairs 0 .. 8*k0 - 1.  V uses the 128-byte-swizzled MN-major layout
// (64-dim panels of 128 keys), P the same no-swizzle K-major layout as Q.
//
// TMEM columns: S double buffer at [0,128) and [128,256), O at [256, 256+D).
#pragma once

#include "device_util.cuh"

namespace wpattn {

constexpr int kBM = 128;              // query rows per CTA
constexpr int kBN = 128;              // keys per tile
constexpr int kPrefillThreads = 192;  // 4 softmax warps + producer + MMA

struct PrefillParams {
  uint16_t* out;      // [B, Nq, Hq, D] bf16
  float* lse;         // [B, Hq, Nq] or null
  int B, Nq, Nk, Hq, Hkv, G;
  int num_qtiles;
  int64_t q_pos0, k_pos0;
  float scale_log2;   // softmax scale * log2(e)
  int64_t T[64];      // per-pair thresholds (nondecreasing)
};

template <int D>
struct PrefillSmem {
  static constexpr int NS = (D == 64) ? 3 : 2;       // K/V ring depth
  static constexpr int TILE = kBM * D * 2;           // one Q, K or V tile in bytes
  static constexpr int PBUF = kBM * kBN * 2;         // one P tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE;
  static constexpr int OFF_V = OFF_K + NS * TILE;
  static constexpr int OFF_P = OFF_V + NS * TILE;
  static constexpr int OFF_BAR = OFF_P + 2 * PBUF;
  // barriers: q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS],
  //           s_full[2], s_free[2], p_full[2], pv_done[2]
  static constexpr int NBAR = 1 + 4 * NS + 8;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_TMEM + 16;
  static constexpr int ALLOC = BYTES + 1024;          // slack for 1024-byte alignment
};

__device__ __forceinline__ int dev_pmin(const int64_t* T, int P, int64_t d) {
  int lo = 0, hi = P;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (T[mid] < d) lo = mid + 1; else hi = mid;
  }
  return lo;
}

template <int D>
__global__ void __launch_bounds__(kPrefillThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ PrefillParams p) {
  using L = PrefillSmem<D>;
  constexpr int NS = L::NS;
  constexpr int P = D / 2;
  constexpr int KS = D / 16;          // k-steps of the QK contraction (8 pairs each)
  constexpr int PANEL = kBM * 16;     // bytes of one 8-dim column panel
  constexpr uint32_t TMEM_S = 0, TMEM_O = 256;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + L::OFF_Q;
  const uint32_t sK = sbase + L::OFF_K;
  const uint32_t sV = sbase + L::OFF_V;
  const uint32_t sP = sbase + L::OFF_P;
  const uint32_t bar = sbase + L::OFF_BAR;
  const uint32_t q_full = bar;
  auto k_full = [&](int s) { return bar + 8 * (1 + s); };
  auto k_empty = [&](int s) { return bar + 8 * (1 + NS + s); };
  auto v_full = [&](int s) { return bar + 8 * (1 + 2 * NS + s); };
  auto v_empty = [&](int s) { return bar + 8 * (1 + 3 * NS + s); };
  auto s_full = [&](int b) { return bar + 8 * (1 + 4 * NS + b); };
  auto s_free = [&](int b) { return bar + 8 * (3 + 4 * NS + b); };
  auto p_full = [&](int b) { return bar + 8 * (5 + 4 * NS + b); };
  auto pv_done = [&](int b) { return bar + 8 * (7 + 4 * NS + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = p.num_qtiles - 1 - blockIdx.x;  // longest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / p.G;

  // key tiles this query tile sees: keys at positions <= its last row
  const int64_t i_min = p.q_pos0 + (int64_t)kBM * qt;
  const int64_t i_max = p.q_pos0 + (int64_t)min(kBM * qt + kBM - 1, p.Nq - 1);
  const int nkt = (p.Nk + kBN - 1) / kBN;
  int n_tiles = 0;
  int kt_last = -1;
  if (i_max >= p.k_pos0 && p.Nk > 0) {
    const int64_t last = (i_max - p.k_pos0) / kBN;
    kt_last = (int)(last < (int64_t)(nkt - 1) ? last : (int64_t)(nkt - 1));
    n_tiles = kt_last + 1;
  }
  // first active k-step of tile j: pairs active at the tile's smallest distance
  auto tile_k0 = [&](int j) -> int {
    const int64_t kp0 = p.k_pos0 + (int64_t)kBN * (kt_last - j);
    int64_t dlo = i_min - (kp0 + kBN - 1);
    if (dlo < 0) dlo = 0;
    return dev_pmin(p.T, P, dlo) / 8;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 5);  // MMA commit + 4 softmax warps (they read K for corrections)
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(s_free(i), 4);
      mbar_init(p_full(i), 4);
      mbar_init(pv_done(i), 1);
    }
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_tiles > 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      mbar_arrive_expect_tx(q_full, L::TILE);
      for (int c = 0; c < D / 8; ++c)
        tma_load_4d(sQ + c * PANEL, &tmQ, q_full, 8 * c, kBM * qt, h, b);
      for (int j = 0; j < n_tiles; ++j) {
        const int kt = kt_last - j;
        const int s = j % NS;
        const uint32_t ph = (j / NS) & 1;
        if (j >= NS && !mbar_wait(k_empty(s), ph ^ 1)) break;
        mbar_arrive_expect_tx(k_full(s), L::TILE);
        for (int c = 0; c < D / 8; ++c)
          tma_load_4d(sK + s * L::TILE + c * PANEL, &tmK, k_full(s), 8 * c, kBN * kt, kvh, b);
        if (j >= NS && !mbar_wait(v_empty(s), ph ^ 1)) break;
        mbar_arrive_expect_tx(v_full(s), L::TILE);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sV + s * L::TILE + c * (kBN * 128), &tmV, v_full(s), 64 * c, kBN * kt, kvh, b);
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idesc_qk = make_idesc_bf16(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_pv = make_idesc_bf16(kBM, D, 0, 1);
      constexpr uint32_t LBO_QK = (D / 16) * PANEL;  // first half -> second half of a pair
      bool ok = mbar_wait(q_full, 0);
      int last_pv = -1;
      auto issue_pv = [&](int i) -> bool {
        if (!mbar_wait(p_full(i & 1), (i >> 1) & 1)) return false;
        if (!mbar_wait(v_full(i % NS), (i / NS) & 1)) return false;
        tc_fence_after();
        const uint32_t pbuf = sP + (i & 1) * L::PBUF;
        const uint32_t vbuf = sV + (i % NS) * L::TILE;
#pragma unroll
        for (int ks = 0; ks < kBN / 16; ++ks) {
          const uint64_t ad = make_sdesc(pbuf + ks * 2 * PANEL, PANEL, 128, 0);
          const uint64_t bd = make_sdesc(vbuf + ks * 2048, kBN * 128, 1024, 2);
          umma_ss(tmem + TMEM_O, ad, bd, idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(pv_done(i & 1));
        umma_commit(v_empty(i % NS));
        last_pv = i;
        return true;
      };
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % NS;
        if (!mbar_wait(k_full(s), (j / NS) & 1)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(s_free(j & 1), ((j - 2) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const int k0 = tile_k0(j);
        const uint32_t kbuf = sK + s * L::TILE;
        for (int ks = k0; ks < KS; ++ks) {
          const uint64_t ad = make_sdesc(sQ + ks * PANEL, LBO_QK, 128, 0);
          const uint64_t bd = make_sdesc(kbuf + ks * PANEL, LBO_QK, 128, 0);
          umma_ss(tmem + TMEM_S + (j & 1) * kBN, ad, bd, idesc_qk, ks > k0 ? 1u : 0u);
        }
        umma_commit(s_full(j & 1));
        umma_commit(k_empty(s));
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(n_tiles - 1);
      // do not release TMEM while an MMA may still write it
      if (last_pv >= 0) mbar_wait(pv_done(last_pv & 1), (last_pv >> 1) & 1);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int r = threadIdx.x;               // row within the tile = TMEM lane
    const int t = kBM * qt + r;
    const int64_t i_pos = i_min + r;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const uint8_t* smem_q = smem + L::OFF_Q;
    float m_ref = -INFINITY;   // max used as the exponent reference of O and l (log2 units)
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int kt = kt_last - j;
      const int s = j % NS;
      const int bsel = j & 1;
      const int64_t kp0 = p.k_pos0 + (int64_t)kBN * kt;
      const int64_t d_row = i_pos - kp0;     // distance to the tile's first key
      const int k0 = tile_k0(j);

      if (!mbar_wait(s_full(bsel), (j >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      float sc[kBN];
#pragma unroll
      for (int cc = 0; cc < kBN / 32; ++cc)
        tmem_ld32(lane_base + TMEM_S + bsel * kBN + 32 * cc,
                  *reinterpret_cast<float(*)[32]>(&sc[32 * cc]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free(bsel));

      if (k0 >= KS) {
#pragma unroll
        for (int c = 0; c < kBN; ++c) sc[c] = 0.f;   // every pair pruned: score 0
      } else {
        // pairs 8*k0 .. p_min(d)-1 went through the MMA but are pruned at d
        const int pm_row = d_row > 0 ? dev_pmin(p.T, P, d_row) : 0;
        const int pc_lo = 8 * k0;
        const int pc_hi = __reduce_max_sync(0xffffffffu, pm_row);
        if (pc_hi > pc_lo) {
          if (!mbar_wait(k_full(s), (j / NS) & 1)) { ok = false; break; }
          const uint8_t* kb = smem + L::OFF_K + s * L::TILE;
          for (int pp = pc_lo; pp < pc_hi; ++pp) {
            int64_t lim64 = d_row - p.T[pp];        // columns c < lim have d > T_pp
            const int lim = (int)(lim64 < 0 ? 0 : (lim64 > kBN ? kBN : lim64));
            if (!__any_sync(0xffffffffu, lim > 0)) continue;
            const int off_lo = (pp >> 3) * PANEL + (pp & 7) * 2;
            const int off_hi = (P / 8 + (pp >> 3)) * PANEL + (pp & 7) * 2;
            const float qa = __uint_as_float((uint32_t)(*reinterpret_cast<const uint16_t*>(smem_q + off_lo + r * 16)) << 16);
            const float qb = __uint_as_float((uint32_t)(*reinterpret_cast<const uint16_t*>(smem_q + off_hi + r * 16)) << 16);
#pragma unroll
            for (int c = 0; c < kBN; ++c) {
              if (c < lim) {
                const float ka = __uint_as_float((uint32_t)(*reinterpret_cast<const uint16_t*>(kb + off_lo + c * 16)) << 16);
                const float kb2 = __uint_as_float((uint32_t)(*reinterpret_cast<const uint16_t*>(kb + off_hi + c * 16)) << 16);
                sc[c] -= fmaf(qa, ka, qb * kb2);
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(k_empty(s));

      // causal mask (d < 0) and the ragged key tail
      const int64_t dlo_tile = i_min - (kp0 + kBN - 1);
      const bool tail = (int64_t)kBN * kt + kBN > p.Nk;
      if (dlo_tile < 0 || tail) {
        int64_t cmax = d_row;                                 // last column with d >= 0
        const int64_t cnk = (int64_t)p.Nk - 1 - (int64_t)kBN * kt;  // last real key
        if (cnk < cmax) cmax = cnk;
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c > cmax) sc[c] = -INFINITY;
      }

      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBN; ++c) mt = fmaxf(mt, sc[c]);
      mt *= p.scale_log2;

      // lazy rescale: move the reference only when the max grew by > 8 (x256)
      float f = 1.f;
      bool resc = false;
      if (j == 0) {
        m_ref = mt;
      } else if (mt > m_ref + 8.f) {
        f = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - mt);
        m_ref = mt;
        resc = true;
      }
      if (__any_sync(0xffffffffu, resc)) {
        if (!mbar_wait(pv_done((j - 1) & 1), ((j - 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          float o[32];
          tmem_ld32(lane_base + TMEM_O + 32 * cc, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= f;
          tmem_st32(lane_base + TMEM_O + 32 * cc, o);
        }
        tmem_st_wait();
      }
      l_run *= f;

      // P buffer bsel was last read by PV(j-2)
      if (j >= 2 && !mbar_wait(pv_done(bsel), ((j - 2) >> 1) & 1)) { ok = false; break; }
      const float msafe = (m_ref == -INFINITY) ? 0.f : m_ref;
      uint8_t* pb = smem + L::OFF_P + bsel * L::PBUF + r * 16;
      float rowsum = 0.f;
#pragma unroll
      for (int kc = 0; kc < kBN / 8; ++kc) {
        float pv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          pv[e] = ex2_approx(fmaf(sc[8 * kc + e], p.scale_log2, -msafe));
          rowsum += pv[e];
        }
        uint4 w;
        w.x = pack_bf16x2(pv[0], pv[1]);
        w.y = pack_bf16x2(pv[2], pv[3]);
        w.z = pack_bf16x2(pv[4], pv[5]);
        w.w = pack_bf16x2(pv[6], pv[7]);
        *reinterpret_cast<uint4*>(pb + kc * PANEL) = w;
      }
      l_run += rowsum;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full(bsel));
    }

    // epilogue: O / l
    const bool row_ok = t < p.Nq;
    uint16_t* orow = p.out + (((size_t)b * p.Nq + t) * p.Hq + h) * D;
    if (ok && n_tiles > 0) {
      const int last = n_tiles - 1;
      ok = mbar_wait(pv_done(last & 1), (last >> 1) & 1);
      tc_fence_after();
    }
    const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      float o[32];
      if (n_tiles > 0) {
        tmem_ld32(lane_base + TMEM_O + 32 * cc, o);
        tmem_ld_wait();
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = (n_tiles > 0) ? o[e] * inv : 0.f;
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
    if (row_ok && p.lse)
      p.lse[((size_t)b * p.Hq + h) * p.Nq + t] =
          (l_run > 0.f) ? (m_ref + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, 512);
}

}  // namespace wpattn
