// Split-KV decode for windowed attention (one new query per sequence).
//
// "ATFlash: Per-RoPE-Wavelength Attention Windows", Abstract: the window is
// a slice of the query-key contraction axis ported into a FlashInfer-style
// decode kernel, which then reads K only over the active head-dim slice of
// each key block.  Each CTA covers one (sequence, kv head, key range) and all
// the query heads of the GQA group (up to GC at a time), so a K/V byte is
// read once for the group.  A producer warp streams blocks of 32 keys of K
// and V through a shared-memory ring with TMA; each block is consumed by one
// of four compute warps, which run both contractions on warp-level tensor-
// core MMAs (mma.sync m16n8k16): S^T = K Q^T over the groups of 8 pairs still
// kept in the block, then O^T += V^T P^T.  With the pair-major K cache only
// the slabs of the block's kept groups are loaded (1 KB each).  In the
// [B, L, Hkv, D] layout (contiguous or paged) whole K rows are loaded: each
// 128-byte half of a row holds one half of every pair, DRAM moves whole half
// rows whatever part of them is asked for (measured with 32-byte column
// copies: the same DRAM bytes as whole rows), and the kept slice reaches
// into both halves at every distance.  A second kernel merges the key ranges
// by their log-sum-exp.
#pragma once

#include "device_util.cuh"
#include "rope_kernels.cuh"

namespace wpattn {

constexpr int kDecodeMaxB = 1024;
constexpr int kDecodeThreads = 128;

struct DecodeParams {
  const uint16_t* q;   // [B, Hq, D]
  const uint16_t* k;   // [B, Lmax, Hkv, D]
  const uint16_t* v;   // [B, Lmax, Hkv, D]
  float* part;         // [B, Hq, S, D + 2]: unnormalised o, running max (log2 units), sum
  uint16_t* out;       // [B, Hq, D]
  float* lse;          // [B, Hq] natural log, or null
  int64_t Lmax;
  int B, Hq, Hkv, G;   // G = Hq / Hkv
  int S;               // key ranges per sequence
  int hchunks;         // ceil(G / GC)
  float scale_log2;    // softmax scale * log2(e)
  int T[64];           // per-pair thresholds, clamped to int32
  // paged cache (block_table != null): k and v are page pools
  // [num_pages, page_size, Hkv, D]; key j of sequence b is row j % page_size of
  // page block_table[b * max_pages + j / page_size]
  const int32_t* block_table;
  int max_pages, page_size, num_pages;
  // explicit key positions (k_pos != null): key j of sequence b sits at
  // k_pos[b * k_pos_stride + j]; otherwise at position j
  const int32_t* k_pos;
  int64_t k_pos_stride;
  int kv_len[kDecodeMaxB];
  int q_pos[kDecodeMaxB];  // position of each sequence's query
  // rope_q: q arrives before its RoPE rotation; the kernel turns it by
  // q_pos * theta_p (rounded to bf16, as a model would store it) on load
  int rope_q;
  double theta[64];
};

// Shared-memory ring of the split kernel: blocks of KB keys of K and V in
// the 128-byte-swizzled layout TMA writes (64-dim panels, row = key), plus
// the query heads, the thresholds and each warp's p row.
constexpr int kDecodeComputeWarps = 4;

template <int D>
struct DecodeSmem {
  static constexpr int KB = 32;                        // keys per block (one per lane)
  // ring depth (blocks in flight): a multiple of the compute warps, so that
  // stage s is only ever consumed by warp s mod W and a warp never waits on a
  // phase of a stage whose previous phase belongs to another warp (a parity
  // wait cannot tell phase k from phase k - 2)
  static constexpr int NS = (D == 64) ? 8 : 4;
  static constexpr int PANEL = KB * 128;               // one 64-dim panel of a block
  static constexpr int TILE = KB * D * 2;              // K or V block
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = NS * TILE;
  static constexpr int OFF_Q = 2 * NS * TILE;          // [8 heads][D] bf16 query heads (zero past the CTA's)
  static constexpr int OFF_T = OFF_Q + 8 * D * 4;      // thresholds (64 x int32)
  static constexpr int OFF_P = OFF_T + 64 * 4;         // [warps][8 heads][KB] fp32 weights
  static constexpr int OFF_BAR = OFF_P + kDecodeComputeWarps * 8 * KB * 4;  // full[NS], empty[NS]
  static constexpr int BYTES = OFF_BAR + 2 * NS * 8;
  static constexpr int ALLOC = BYTES + 1024;           // slack to align the ring to 1024 bytes
};

// 16 bytes of a K or V row from the swizzled ring: row r (key within the
// block), 16-byte chunk c of the head dim.  Eight consecutive rows put a
// given chunk in eight different 16-byte bank groups.
template <int D>
__device__ __forceinline__ uint4 ring_chunk(const uint8_t* tile, int r, int c) {
  using L = DecodeSmem<D>;
  return *reinterpret_cast<const uint4*>(tile + (c >> 3) * L::PANEL + r * 128 +
                                         (((c & 7) ^ (r & 7)) << 4));
}

// Work split inside a CTA: the producer warp streams blocks of 32 keys; block
// i goes to compute warp i mod 4, which computes its scores for every query
// head of the CTA over the block's kept groups, runs the online softmax and
// accumulates O^T, all in registers (the query heads fill the n = 8 side of
// the MMAs).  The warps merge through shared memory at the end.
//
// PM (pair-major K cache): K is stored as [B, Hkv, D/16, Lmax, 16], slab g
// holding dims 8g..8g+7 and P+8g..P+8g+7 of every key (the 8 pairs of one
// group).  The producer then loads only the slabs still kept for the block
// (1 KB each, from the first kept group on), so the window cuts DRAM bytes;
// in the ring, slab g of a block sits at 1 KB * g, key r at 32 bytes * r.
template <int D, int GC, bool PM>
__global__ void __launch_bounds__((kDecodeComputeWarps + 1) * 32, GC <= 4 ? 3 : 2)
decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ DecodeParams p) {
  using L = DecodeSmem<D>;
  constexpr int KB = L::KB, NS = L::NS, W = kDecodeComputeWarps;
  constexpr int P = D / 2;
  constexpr int NG = P / 8;               // groups of 8 pairs (16 dims: 8 in each half)
  constexpr int NMT = D / 16;             // PV: 16-dim row tiles of O^T
  constexpr uint32_t FULL = 0xffffffffu;
  static_assert(W * GC * D * 4 <= 2 * NS * L::TILE, "merge buffer must fit in the ring");
  static_assert(NS % W == 0, "each ring stage must belong to one compute warp");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the swizzled ring starts on a 1024-byte boundary of the shared window
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ float sm_m[W][GC];
  __shared__ float sm_l[W][GC];
  // the merge's partial outputs reuse the ring once every block is consumed
  float (*sm_o)[GC][D] = reinterpret_cast<float (*)[GC][D]>(smem);
  uint16_t* qb = reinterpret_cast<uint16_t*>(smem + L::OFF_Q);
  int* sT = reinterpret_cast<int*>(smem + L::OFF_T);

  const uint32_t sbase = smem_u32(smem);
  auto full = [&](int s) { return sbase + L::OFF_BAR + 8 * s; };
  auto empty = [&](int s) { return sbase + L::OFF_BAR + 8 * (NS + s); };

  const int split = blockIdx.x;
  const int kvh = blockIdx.y / p.hchunks;
  const int hc = blockIdx.y % p.hchunks;
  const int b = blockIdx.z;
  const int h0 = kvh * p.G + hc * GC;
  const int nh = min(GC, p.G - hc * GC);
  const int Lb = p.kv_len[b];
  const int chunk = ((Lb + p.S - 1) / p.S + 63) / 64 * 64;
  const int j_begin = split * chunk;
  const int j_end = min(Lb, j_begin + chunk);
  const int nblk = j_end > j_begin ? (j_end - j_begin + KB - 1) / KB : 0;
  const int qpos = p.q_pos[b];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool paged = !PM && p.block_table != nullptr;
  // first group of 8 pairs kept for some key of the block starting at j0:
  // groups whose largest threshold is below the block's smallest distance
  // (that of its last real key) are pruned for every key of the block
  auto first_kept_group = [&](int j0) -> int {
    const int dmin = qpos - (min(j0 + KB, j_end) - 1);
    int g0 = 0;
    while (g0 < NG && sT[8 * g0 + 7] < dmin) ++g0;
    return g0;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);   // the one compute warp that owns the block
    }
    fence_barrier_init();
  }
  if (threadIdx.x < 64) sT[threadIdx.x] = p.T[threadIdx.x];
  if (p.rope_q) {
    for (int idx = threadIdx.x; idx < 8 * P; idx += blockDim.x) {
      const int hh = idx / P, pp = idx % P;
      float y0 = 0.f, y1 = 0.f;
      if (hh < nh) {
        const uint16_t* qr = p.q + ((size_t)b * p.Hq + h0 + hh) * D;
        float c, sn;
        rope_cos_sin(qpos, p.theta[pp], c, sn);
        rope_pair_bf16(bf16lo_to_f32(qr[pp]), bf16lo_to_f32(qr[pp + P]), c, sn, y0, y1);
      }
      qb[hh * D + pp] = static_cast<uint16_t>(__float_as_uint(y0) >> 16);   // y0, y1 are bf16 values
      qb[hh * D + pp + P] = static_cast<uint16_t>(__float_as_uint(y1) >> 16);
    }
  } else {
    for (int idx = threadIdx.x; idx < 8 * D; idx += blockDim.x) {
      const int hh = idx / D, e = idx % D;
      qb[idx] = hh < nh ? p.q[((size_t)b * p.Hq + h0 + hh) * D + e] : static_cast<uint16_t>(0);
    }
  }
  __syncthreads();

  if (warp == W) {
    // ------------------------------------------------------------ producer
    // The whole warp walks the blocks (lane 0 issues the copies) so that, for
    // a paged cache, the lanes can fetch 32 page numbers at a time.
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
    }
    // paged: rows per copy (one page, at most one block), copies per block
    const int R = p.block_table ? min(p.page_size, KB) : KB;
    const int U = KB / R;
    // page of copy unit u (R rows from j_begin + u * R): lane l holds unit
    // 32 k + l of the current batch k and, loaded one batch ahead so that its
    // latency is hidden, of the next
    auto fetch_page = [&](int unit) -> int {
      const long long jl = j_begin + static_cast<long long>(unit) * R;
      if (!p.block_table || jl >= j_end) return 0;
      const int pg = p.block_table[(size_t)b * p.max_pages + static_cast<int>(jl / p.page_size)];
      if (pg < 0 || pg >= p.num_pages) {
        record_status(6 /* WPATTN_EINDEX */);
        return 0;                         // read a real page; the output is flagged
      }
      return pg;
    };
    int my_page = 0, next_page = 0;
    if (paged) {
      my_page = fetch_page(lane);
      next_page = fetch_page(32 + lane);
    }
    // addressing of the next block, worked out while its ring stage drains
    int pg[4], row0 = 0, nsub = 0;
    auto plan_block = [&](int i) {
      const int unit0 = i * U;            // copy units of this CTA's range, R rows each
      if (unit0 > 0 && (unit0 & 31) == 0) {
        my_page = next_page;
        next_page = fetch_page(unit0 + 32 + lane);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) pg[u] = __shfl_sync(FULL, my_page, (unit0 + u) & 31);
      const int j0 = j_begin + i * KB;
      row0 = R < KB ? 0 : j0 % p.page_size;  // R < KB: one page per unit, from its row 0
      nsub = (min(j0 + KB, j_end) - j0 + R - 1) / R;
    };
    if (paged && nblk > 0) plan_block(0);
    // pair-major: first slab of the next block, found while its stage drains
    int g0_next = (PM && nblk > 0) ? first_kept_group(j_begin) : 0;
    int issued = 0;           // blocks whose copies were issued
    bool ok_prod = true;
    for (int i = 0; i < nblk; ++i) {
      const int s = i % NS;
      if (i >= NS && !__all_sync(FULL, mbar_wait(empty(s), ((i / NS) & 1) ^ 1))) {
        ok_prod = false;
        break;
      }
      const int j0 = j_begin + i * KB;
      if (paged) {
        if (lane == 0) {
          mbar_arrive_expect_tx(full(s), nsub * R * D * 2 * 2);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (u >= nsub) break;
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              const uint32_t off = s * L::TILE + c * L::PANEL + u * R * 128;
              tma_load_4d(sbase + L::OFF_K + off, &tmK, full(s), 64 * c, row0, kvh, pg[u]);
              tma_load_4d(sbase + L::OFF_V + off, &tmV, full(s), 64 * c, row0, kvh, pg[u]);
            }
          }
        }
        issued = i + 1;
        if (i + 1 < nblk) plan_block(i + 1);
        continue;
      }
      if (lane == 0) {
        const int g0 = g0_next;
        if (PM) {
          mbar_arrive_expect_tx(full(s), (NG - g0) * KB * 32 + L::TILE);
          for (int g = g0; g < NG; ++g)
            tma_load_4d(sbase + L::OFF_K + s * L::TILE + g * KB * 32, &tmK, full(s), 0, j0, kvh * NG + g, b);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sbase + L::OFF_V + s * L::TILE + c * L::PANEL, &tmV, full(s), 64 * c, j0, kvh, b);
        } else {
          mbar_arrive_expect_tx(full(s), 2 * L::TILE);
          for (int c = 0; c < D / 64; ++c) {
            tma_load_4d(sbase + L::OFF_K + s * L::TILE + c * L::PANEL, &tmK, full(s), 64 * c, j0, kvh, b);
            tma_load_4d(sbase + L::OFF_V + s * L::TILE + c * L::PANEL, &tmV, full(s), 64 * c, j0, kvh, b);
          }
        }
      }
      issued = i + 1;
      if (PM && i + 1 < nblk) g0_next = first_kept_group(j0 + KB);
    }
    if (!ok_prod) {
      // A wait ran out: copies issued into the ring may still be landing.
      // Wait (bounded) for the fill of every stage's last issued block before
      // the CTA can leave; older blocks completed before their stage was reused.
      for (int i = max(0, issued - NS); i < issued; ++i) (void)mbar_wait(full(i % NS), (i / NS) & 1);
    }
    return;  // the producer takes no part in the merge below
  }

  // ---------------------------------------------------------------- compute
  // PV on the tensor cores, per warp: O^T [D x 8 heads] += V^T [D x 16 keys] .
  // P^T [16 keys x 8 heads], m16n8k16 steps (the heads of a CTA, at most 8,
  // fill the n = 8 side).  Lane (gid = lane / 4, tig = lane % 4) holds, for row
  // tile mt, dims 16 mt + gid and 16 mt + gid + 8 of heads 2 tig and 2 tig + 1.
  const int gid = lane >> 2, tig = lane & 3;
  float* pw = reinterpret_cast<float*>(smem + L::OFF_P) + warp * 8 * KB;  // this warp's p rows
  float m[GC], l[GC];
  float oacc[NMT][4];
#pragma unroll
  for (int hh = 0; hh < GC; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.f;
  }
#pragma unroll
  for (int mt = 0; mt < NMT; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) oacc[mt][e] = 0.f;
  // lane's row address of matrix ldm_m = lane / 8 in the ldmatrix of (row tile
  // mt, key step ks): key 16 ks + 8 (ldm_m >> 1) + lane % 8, dims chunk
  // 2 mt + (ldm_m & 1)
  const int ldm_key = 8 * ((lane >> 3) >> 1) + (lane & 7);
  const int ldm_chunk = (lane >> 3) & 1;

  for (int i = warp; i < nblk; i += W) {
    const int s = i % NS;
    const int j0 = j_begin + i * KB;
    const int j = j0 + lane;              // this lane's key
    // explicit positions: fetched before the wait so the load overlaps it
    int kpos = j;
    if (p.k_pos && j < j_end) kpos = p.k_pos[(size_t)b * p.k_pos_stride + j];
    // contiguous positions: the block's first kept group is known before its data
    int g0 = p.k_pos ? 0 : first_kept_group(j0);
    if (!__all_sync(FULL, mbar_wait(full(s), (i / NS) & 1))) break;
    const uint8_t* kt = smem + L::OFF_K + s * L::TILE;
    const uint8_t* vt = smem + L::OFF_V + s * L::TILE;
    bool valid = j < j_end;
    int dist = qpos - kpos;
    if (p.k_pos) {
      if (valid && kpos < 0) {
        record_status(6 /* WPATTN_EINDEX */);
        kpos = qpos + 1;                  // treated as a future key
        dist = -1;
      }
      valid = valid && kpos <= qpos;      // keys after the query are causally excluded
      // smallest distance over the block's attended keys (positions need not be sorted)
      const int dmin = __reduce_min_sync(FULL, valid ? dist : 0x7fffffff);
      while (g0 < NG && sT[8 * g0 + 7] < dmin) ++g0;
    }

    // ---- scores on the tensor cores: S^T [32 keys x 8 heads] = K . Q^T over
    // the kept groups g0 .. NG-1, one m16n8k16 step per (16 keys, group).  A
    // group's k-step is its 16 dims: 8g..8g+7, then P+8g..P+8g+7.  Lane (gid,
    // tig) holds the A elements of keys gid (+8) and pairs 8g + 2 tig (+1);
    // where the window prunes a pair at a key's distance the element is zeroed.
    float sacc[KB / 16][4];
#pragma unroll
    for (int mt = 0; mt < KB / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[mt][e] = 0.f;
    {
      int dk[KB / 8];                     // distances of keys gid, gid + 8, gid + 16, gid + 24
#pragma unroll
      for (int r = 0; r < KB / 8; ++r) dk[r] = __shfl_sync(FULL, dist, gid + 8 * r);
      const uint16_t* qrow = qb + gid * D;
      // this lane's ldmatrix row: matrix lane / 8 = (keys + 8 (lane / 8 & 1), half lane / 16)
      const int lkey = 8 * ((lane >> 3) & 1) + (lane & 7);
      const int lhalf = lane >> 4;
#pragma unroll 1
      for (int g = g0; g < NG; ++g) {
        // B = Q^T: dims 8g + 2 tig (+1) and P + 8g + 2 tig (+1) of head gid
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(qrow + 8 * g + 2 * tig);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(qrow + P + 8 * g + 2 * tig);
        const bool prune = __any_sync(FULL, dist > sT[8 * g]);
        const int T0 = sT[8 * g + 2 * tig], T1 = sT[8 * g + 2 * tig + 1];
#pragma unroll
        for (int mt = 0; mt < KB / 16; ++mt) {
          const int key = 16 * mt + lkey;
          uint32_t addr;
          if (PM) {
            addr = smem_u32(kt) + g * KB * 32 + key * 32 + lhalf * 16;
          } else {
            const int ch = lhalf ? NG + g : g;
            addr = smem_u32(kt) + (ch >> 3) * L::PANEL + key * 128 + (((ch & 7) ^ (key & 7)) << 4);
          }
          uint32_t a0, a1, a2, a3;
          ldsm_x4(addr, a0, a1, a2, a3);
          if (prune) {
            const int d0 = dk[2 * mt], d1 = dk[2 * mt + 1];
            const uint32_t m0 = (d0 > T0 ? 0u : 0x0000FFFFu) | (d0 > T1 ? 0u : 0xFFFF0000u);
            const uint32_t m1 = (d1 > T0 ? 0u : 0x0000FFFFu) | (d1 > T1 ? 0u : 0xFFFF0000u);
            a0 &= m0; a2 &= m0; a1 &= m1; a3 &= m1;
          }
          mma_16816_bf16(sacc[mt], a0, a1, a2, a3, b0, b1);
        }
      }
    }
    // S^T through the warp's p rows (free until the softmax writes them): each
    // lane then holds its own key's scores for every head, in log2 units
    {
      float* ssc = pw;                    // [32 keys][8 heads]
#pragma unroll
      for (int mt = 0; mt < KB / 16; ++mt) {
        *reinterpret_cast<float2*>(ssc + (16 * mt + gid) * 8 + 2 * tig) = make_float2(sacc[mt][0], sacc[mt][1]);
        *reinterpret_cast<float2*>(ssc + (16 * mt + gid + 8) * 8 + 2 * tig) = make_float2(sacc[mt][2], sacc[mt][3]);
      }
    }
    __syncwarp();
    float sc[GC];
#pragma unroll
    for (int hh = 0; hh < GC; ++hh) sc[hh] = pw[lane * 8 + hh] * p.scale_log2;
    __syncwarp();                         // every lane has its scores before p overwrites them

    // ---- online softmax over the block (warp-wide max per head)
    float corr_h[GC];
#pragma unroll
    for (int hh = 0; hh < GC; ++hh) {
      const float sv = valid ? sc[hh] : -INFINITY;
      float bm = sv;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(FULL, bm, off));
      const float mn = fmaxf(m[hh], bm);
      float pv = 0.f;
      corr_h[hh] = 1.f;
      if (mn != -INFINITY) {
        const float corr = (m[hh] == -INFINITY) ? 0.f : ex2_approx(m[hh] - mn);
        pv = ex2_approx(sv - mn);
        l[hh] = l[hh] * corr + pv;        // this lane's key only; summed over lanes at the end
        corr_h[hh] = corr;
        m[hh] = mn;
      }
      pw[hh * KB + lane] = pv;
    }
    __syncwarp();

    // ---- O^T = O^T * corr + V^T P^T on the tensor cores
    {
      // this lane's heads 2 tig, 2 tig + 1 (1 where they are past the CTA's heads)
      float ca = 1.f, cb = 1.f;
      bool moved = false;
#pragma unroll
      for (int hh = 0; hh < GC; ++hh) {
        moved |= corr_h[hh] != 1.f;
        if (hh == 2 * tig) ca = corr_h[hh];
        if (hh == 2 * tig + 1) cb = corr_h[hh];
      }
      if (moved) {
#pragma unroll
        for (int mt = 0; mt < NMT; ++mt) {
          mul2(oacc[mt][0], oacc[mt][1], oacc[mt][0], oacc[mt][1], ca, cb);
          mul2(oacc[mt][2], oacc[mt][3], oacc[mt][2], oacc[mt][3], ca, cb);
        }
      }
    }
    // keys past the sequence end hold anything (a cache may keep NaN there):
    // their V elements are zeroed before the product, their p is 0
    const int nvalid = min(KB, j_end - j0);
#pragma unroll
    for (int ks = 0; ks < KB / 16; ++ks) {
      if (16 * ks >= nvalid) break;
      // B = P^T: keys 16 ks + 2 tig (+1) and + 8, head gid (0 past the CTA's heads)
      uint32_t b0 = 0u, b1 = 0u;
      if (gid < GC) {
        const float2 x0 = *reinterpret_cast<const float2*>(pw + gid * KB + 16 * ks + 2 * tig);
        const float2 x1 = *reinterpret_cast<const float2*>(pw + gid * KB + 16 * ks + 8 + 2 * tig);
        b0 = pack_bf16x2(x0.x, x0.y);
        b1 = pack_bf16x2(x1.x, x1.y);
      }
      const int key = 16 * ks + ldm_key;
      // element masks of the A registers: (key 2 tig, 2 tig + 1) and the same + 8
      const int kl = 16 * ks + 2 * tig;
      const uint32_t mlo = (kl < nvalid ? 0x0000FFFFu : 0u) | (kl + 1 < nvalid ? 0xFFFF0000u : 0u);
      const uint32_t mhi = (kl + 8 < nvalid ? 0x0000FFFFu : 0u) | (kl + 9 < nvalid ? 0xFFFF0000u : 0u);
#pragma unroll
      for (int mt = 0; mt < NMT; ++mt) {
        const int chunk = 2 * mt + ldm_chunk;
        const uint32_t addr = smem_u32(vt) + (chunk >> 3) * L::PANEL + key * 128 +
                              (((chunk & 7) ^ (key & 7)) << 4);
        uint32_t a0, a1, a2, a3;
        ldsm_x4_trans(addr, a0, a1, a2, a3);
        a0 &= mlo; a1 &= mlo; a2 &= mhi; a3 &= mhi;
        mma_16816_bf16(oacc[mt], a0, a1, a2, a3, b0, b1);
      }
    }
    __syncwarp();  // the p rows are rewritten by the next block
    if (lane == 0) mbar_arrive(empty(s));
  }

  // combine this warp's lanes' l (one key each)
#pragma unroll
  for (int hh = 0; hh < GC; ++hh) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l[hh] += __shfl_xor_sync(FULL, l[hh], off);
  }

  // merge the warps of this CTA (compute warps only); every block has been
  // consumed, so the ring is free
  asm volatile("bar.sync 1, %0;" ::"n"(W * 32) : "memory");
#pragma unroll
  for (int mt = 0; mt < NMT; ++mt) {
    if (2 * tig < GC) {
      sm_o[warp][2 * tig][16 * mt + gid] = oacc[mt][0];
      sm_o[warp][2 * tig][16 * mt + gid + 8] = oacc[mt][2];
    }
    if (2 * tig + 1 < GC) {
      sm_o[warp][2 * tig + 1][16 * mt + gid] = oacc[mt][1];
      sm_o[warp][2 * tig + 1][16 * mt + gid + 8] = oacc[mt][3];
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int hh = 0; hh < GC; ++hh) {
      sm_m[warp][hh] = m[hh];
      sm_l[warp][hh] = l[hh];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(W * 32) : "memory");
  for (int idx = threadIdx.x; idx < nh * D; idx += W * 32) {
    const int hh = idx / D, e = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w2 = 0; w2 < W; ++w2) M = fmaxf(M, sm_m[w2][hh]);
    float Ls = 0.f, Os = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w2 = 0; w2 < W; ++w2) {
        const float wt = ex2_approx(sm_m[w2][hh] - M);
        Ls += sm_l[w2][hh] * wt;
        Os += sm_o[w2][hh][e] * wt;
      }
    }
    float* rec = p.part + (((size_t)b * p.Hq + h0 + hh) * p.S + split) * (D + 2);
    rec[e] = Os;
    if (e == 0) {
      rec[D] = M;
      rec[D + 1] = Ls;
    }
  }
}

// K cache [B, Lmax, Hkv, D] -> pair-major slabs [B, Hkv, D/16, Lmax, 16]:
// slab g of a key holds dims 8g..8g+7 then D/2+8g..D/2+8g+7 (the 8 pairs of
// group g).  One thread per (batch, kv head, slab, key), in slab order, so
// consecutive threads write consecutive 32-byte rows.
template <int D>
__global__ void __launch_bounds__(256)
kcache_to_pairmajor_kernel(const uint16_t* __restrict__ k, uint16_t* __restrict__ slabs, int64_t Lmax,
                           int B, int Hkv) {
  constexpr int NG = D / 16, P = D / 2;
  const uint64_t idx = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint64_t n = static_cast<uint64_t>(B) * Hkv * NG * static_cast<uint64_t>(Lmax);
  if (idx >= n) return;
  const uint64_t j = idx % static_cast<uint64_t>(Lmax);
  const uint64_t plane = idx / static_cast<uint64_t>(Lmax);   // (b * Hkv + h) * NG + g
  const int g = static_cast<int>(plane % NG);
  const uint64_t bh = plane / NG;                              // b * Hkv + h
  const uint64_t b = bh / Hkv, h = bh % Hkv;
  const uint16_t* row = k + ((b * static_cast<uint64_t>(Lmax) + j) * Hkv + h) * D;
  const uint4 lo = *reinterpret_cast<const uint4*>(row + 8 * g);
  const uint4 hi = *reinterpret_cast<const uint4*>(row + P + 8 * g);
  uint4* dst = reinterpret_cast<uint4*>(slabs + idx * 16);
  dst[0] = lo;
  dst[1] = hi;
}

// Merge the S key ranges of each (sequence, query head): out = sum_s w_s o_s
// / sum_s w_s l_s with w_s = 2^(m_s - max m); lse = ln 2 * (max m + log2 sum).
template <int D>
__global__ void __launch_bounds__(D)
decode_combine_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ float sm[];  // [2 * S]: weights, then l_s
  const int bh = blockIdx.x;
  const int e = threadIdx.x;
  const float* recs = p.part + (size_t)bh * p.S * (D + 2);
  float M = -INFINITY;
  for (int s = e; s < p.S; s += D) M = fmaxf(M, recs[(size_t)s * (D + 2) + D]);
  // block max
  __shared__ float red[D / 32];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if ((e & 31) == 0) red[e >> 5] = M;
  __syncthreads();
  M = red[0];
#pragma unroll
  for (int w = 1; w < D / 32; ++w) M = fmaxf(M, red[w]);
  for (int s = e; s < p.S; s += D) {
    const float ms = recs[(size_t)s * (D + 2) + D];
    const float w = (M == -INFINITY) ? 0.f : ex2_approx(ms - M);
    sm[s] = w;
    sm[p.S + s] = recs[(size_t)s * (D + 2) + D + 1] * w;
  }
  __syncthreads();
  float Ls = 0.f, Os = 0.f;
  for (int s = 0; s < p.S; ++s) {
    Ls += sm[p.S + s];
    Os += sm[s] * recs[(size_t)s * (D + 2) + e];
  }
  const float val = Ls > 0.f ? Os / Ls : 0.f;
  p.out[(size_t)bh * D + e] = static_cast<uint16_t>(pack_bf16x2(val, 0.f) & 0xFFFFu);
  if (p.lse && e == 0)
    p.lse[bh] = Ls > 0.f ? (M + __log2f(Ls)) * 0.69314718055994530942f : -INFINITY;
}

// Merge of R partial results of the same rows (each normalised over its own
// keys, with its log-sum-exp): out = sum_r w_r out_r / sum_r w_r, w_r =
// exp(lse_r - max lse), lse = max lse + ln sum_r w_r.  One block per row,
// one thread per head dim; a row whose parts are all empty gets 0 and -inf.
template <int D>
__global__ void __launch_bounds__(D)
merge_lse_kernel(const uint16_t* __restrict__ outs, const float* __restrict__ lses, int R,
                 int64_t rows, uint16_t* __restrict__ out, float* __restrict__ lse) {
  const int64_t row = blockIdx.x;
  const int e = threadIdx.x;
  float M = -INFINITY;
  for (int r = 0; r < R; ++r) M = fmaxf(M, lses[(size_t)r * rows + row]);
  float W = 0.f, acc = 0.f;
  if (M != -INFINITY) {
    for (int r = 0; r < R; ++r) {
      const float lr = lses[(size_t)r * rows + row];
      const float w = lr == -INFINITY ? 0.f : __expf(lr - M);
      W += w;
      acc += w * bf16lo_to_f32(outs[((size_t)r * rows + row) * D + e]);
    }
  }
  const float val = W > 0.f ? acc / W : 0.f;
  out[(size_t)row * D + e] = static_cast<uint16_t>(pack_bf16x2(val, 0.f) & 0xFFFFu);
  if (lse && e == 0) lse[row] = W > 0.f ? M + __logf(W) : -INFINITY;
}

}  // namespace wpattn
