// Split-KV decode for windowed attention (one new query per sequence).
//
// "ATFlash: Per-RoPE-Wavelength Attention Windows", Abstract: the window is
// a slice of the query-key contraction axis ported into a FlashInfer-style
// decode kernel.  Each CTA covers one (sequence, kv head, key range) and all
// the query heads of the GQA group (up to GC at a time), so a K/V byte is
// read once for the group.  A producer warp streams blocks of 32 keys of K
// and V through a shared-memory ring with TMA (128-byte swizzle); each block
// is consumed by one of four compute warps.  For the scores a lane owns a
// key and walks only the groups of 8 pairs still kept in the block; for
// O += p V a lane owns a 16-byte chunk of the head dim.  In the
// [B, L, Hkv, D] cache layout each half of a K row is one 128-byte line and
// the kept slice touches both, so whole rows move from DRAM either way; the
// window saves arithmetic here, not bytes.  A second kernel merges the key
// ranges by their log-sum-exp.
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

__device__ __forceinline__ uint4 ldg_stream(const void* ptr) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(ptr));
  return r;
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  f[0] = bf16lo_to_f32(u.x); f[1] = bf16hi_to_f32(u.x);
  f[2] = bf16lo_to_f32(u.y); f[3] = bf16hi_to_f32(u.y);
  f[4] = bf16lo_to_f32(u.z); f[5] = bf16hi_to_f32(u.z);
  f[6] = bf16lo_to_f32(u.w); f[7] = bf16hi_to_f32(u.w);
}

// Shared-memory ring of the split kernel: blocks of KB keys of K and V in
// the 128-byte-swizzled layout TMA writes (64-dim panels, row = key), plus
// the pre-scaled query heads, the thresholds and each warp's p row.
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
  static constexpr int OFF_Q = 2 * NS * TILE;          // [8 heads][D] fp32, scaled by scale * log2(e)
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
// i goes to compute warp i mod 4.  For the scores a lane owns one key (its
// whole row): it walks only the groups of 8 pairs that are still kept
// somewhere in the warp's 32 keys, with the query head dims read from shared
// memory (broadcast), so the window removes work and no cross-lane reduction
// is needed.  For O += p V a lane owns one 16-byte chunk of the head dim for
// 32 / (D / 8) keys at a time.
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
  constexpr int TPK = D / 8;              // lanes per key in the PV step (one 16-byte chunk each)
  constexpr int KPW = 32 / TPK;           // keys per PV step
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
  float* qs = reinterpret_cast<float*>(smem + L::OFF_Q);
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
    for (int idx = threadIdx.x; idx < GC * P; idx += blockDim.x) {
      const int hh = idx / P, pp = idx % P;
      float y0 = 0.f, y1 = 0.f;
      if (hh < nh) {
        const uint16_t* qr = p.q + ((size_t)b * p.Hq + h0 + hh) * D;
        float c, sn;
        rope_cos_sin(qpos, p.theta[pp], c, sn);
        rope_pair_bf16(bf16lo_to_f32(qr[pp]), bf16lo_to_f32(qr[pp + P]), c, sn, y0, y1);
      }
      qs[hh * D + pp] = y0 * p.scale_log2;
      qs[hh * D + pp + P] = y1 * p.scale_log2;
    }
  } else {
    for (int idx = threadIdx.x; idx < GC * D; idx += blockDim.x) {
      const int hh = idx / D, e = idx % D;
      qs[idx] = hh < nh ? bf16lo_to_f32(p.q[((size_t)b * p.Hq + h0 + hh) * D + e]) * p.scale_log2 : 0.f;
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
    const bool paged = !PM && p.block_table != nullptr;
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
    for (int i = 0; i < nblk; ++i) {
      const int s = i % NS;
      if (i >= NS && !__all_sync(FULL, mbar_wait(empty(s), ((i / NS) & 1) ^ 1))) break;
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
        if (i + 1 < nblk) plan_block(i + 1);
        continue;
      }
      if (lane == 0) {
        if (PM) {
          const int g0 = g0_next;
          mbar_arrive_expect_tx(full(s), (NG - g0) * KB * 32 + L::TILE);
          for (int g = g0; g < NG; ++g)
            tma_load_4d(sbase + L::OFF_K + s * L::TILE + g * KB * 32, &tmK, full(s), 0, j0, kvh * NG + g, b);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(sbase + L::OFF_V + s * L::TILE + c * L::PANEL, &tmV, full(s), 64 * c, j0, kvh, b);
          if (i + 1 < nblk) g0_next = first_kept_group(j0 + KB);
        } else {
          mbar_arrive_expect_tx(full(s), 2 * L::TILE);
          for (int c = 0; c < D / 64; ++c) {
            tma_load_4d(sbase + L::OFF_K + s * L::TILE + c * L::PANEL, &tmK, full(s), 64 * c, j0, kvh, b);
            tma_load_4d(sbase + L::OFF_V + s * L::TILE + c * L::PANEL, &tmV, full(s), 64 * c, j0, kvh, b);
          }
        }
      }
    }
    return;  // the producer takes no part in the merge below
  }

  // ---------------------------------------------------------------- compute
  const int c = lane % TPK;               // PV: head-dim chunk [8c, 8c+8)
  const int kk = lane / TPK;              // PV: key within a step
  float* pw = reinterpret_cast<float*>(smem + L::OFF_P) + warp * 8 * KB;  // this warp's p rows
  float m[GC], l[GC], o[GC][8];
#pragma unroll
  for (int hh = 0; hh < GC; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[hh][e] = 0.f;
  }

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

    // ---- scores: one key per lane, groups g0 .. NG-1
    float sc[GC];
#pragma unroll
    for (int hh = 0; hh < GC; ++hh) sc[hh] = 0.f;
#pragma unroll 1
    for (int g = g0; g < NG; ++g) {
      float kf[16];
      {
        float a[8], bb[8];
        if (PM) {  // this key's 32-byte row of slab g
          const uint4* row = reinterpret_cast<const uint4*>(kt + g * KB * 32 + lane * 32);
          unpack8(row[0], a);
          unpack8(row[1], bb);
        } else {
          unpack8(ring_chunk<D>(kt, lane, g), a);            // dims 8g .. 8g+7
          unpack8(ring_chunk<D>(kt, lane, NG + g), bb);      // dims P+8g .. P+8g+7
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) { kf[e] = a[e]; kf[8 + e] = bb[e]; }
      }
      // pairs of the group pruned at this key's distance contribute 0
      if (__any_sync(FULL, dist > sT[8 * g])) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (dist > sT[8 * g + e]) { kf[e] = 0.f; kf[8 + e] = 0.f; }
        }
      }
#pragma unroll
      for (int hh = 0; hh < GC; ++hh) {
        const float4* qa = reinterpret_cast<const float4*>(qs + hh * D + 8 * g);
        const float4* qb = reinterpret_cast<const float4*>(qs + hh * D + P + 8 * g);
        const float4 x0 = qa[0], x1 = qa[1], y0 = qb[0], y1 = qb[1];
        float a0 = 0.f, a1 = 0.f;
        fma2(a0, a1, x0.x, x0.y, kf[0], kf[1], a0, a1);
        fma2(a0, a1, x0.z, x0.w, kf[2], kf[3], a0, a1);
        fma2(a0, a1, x1.x, x1.y, kf[4], kf[5], a0, a1);
        fma2(a0, a1, x1.z, x1.w, kf[6], kf[7], a0, a1);
        fma2(a0, a1, y0.x, y0.y, kf[8], kf[9], a0, a1);
        fma2(a0, a1, y0.z, y0.w, kf[10], kf[11], a0, a1);
        fma2(a0, a1, y1.x, y1.y, kf[12], kf[13], a0, a1);
        fma2(a0, a1, y1.z, y1.w, kf[14], kf[15], a0, a1);
        sc[hh] += a0 + a1;
      }
    }

    // ---- online softmax over the block (warp-wide max per head)
#pragma unroll
    for (int hh = 0; hh < GC; ++hh) {
      const float sv = valid ? sc[hh] : -INFINITY;
      float bm = sv;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(FULL, bm, off));
      const float mn = fmaxf(m[hh], bm);
      float pv = 0.f;
      if (mn != -INFINITY) {
        const float corr = (m[hh] == -INFINITY) ? 0.f : ex2_approx(m[hh] - mn);
        pv = ex2_approx(sv - mn);
        l[hh] = l[hh] * corr + pv;        // this lane's key only; summed over lanes at the end
#pragma unroll
        for (int e = 0; e < 8; e += 2) mul2(o[hh][e], o[hh][e + 1], o[hh][e], o[hh][e + 1], corr, corr);
        m[hh] = mn;
      }
      pw[hh * KB + lane] = pv;
    }
    __syncwarp();

    // ---- O += p V: lane (kk, c) takes chunk c of keys kk, kk + KPW, ...
    // (keys past the sequence end are not read: a cache may hold anything there)
    const int nvalid = min(KB, j_end - j0);
#pragma unroll 4
    for (int r = kk; r < nvalid; r += KPW) {
      float vf[8];
      unpack8(ring_chunk<D>(vt, r, c), vf);
#pragma unroll
      for (int hh = 0; hh < GC; ++hh) {
        const float pr = pw[hh * KB + r];
#pragma unroll
        for (int e = 0; e < 8; e += 2) fma2(o[hh][e], o[hh][e + 1], pr, pr, vf[e], vf[e + 1], o[hh][e], o[hh][e + 1]);
      }
    }
    __syncwarp();  // the p rows are rewritten by the next block
    if (lane == 0) mbar_arrive(empty(s));
  }

  // combine this warp's lanes: l over keys (all lanes), o over the KPW key groups
#pragma unroll
  for (int hh = 0; hh < GC; ++hh) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l[hh] += __shfl_xor_sync(FULL, l[hh], off);
#pragma unroll
    for (int off = TPK; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < 8; ++e) o[hh][e] += __shfl_xor_sync(FULL, o[hh][e], off);
    }
  }

  // merge the warps of this CTA (compute warps only); every block has been
  // consumed, so the ring is free
  asm volatile("bar.sync 1, %0;" ::"n"(W * 32) : "memory");
  if (kk == 0) {
#pragma unroll
    for (int hh = 0; hh < GC; ++hh) {
#pragma unroll
      for (int e = 0; e < 8; ++e) sm_o[warp][hh][8 * c + e] = o[hh][e];
      if (c == 0) {
        sm_m[warp][hh] = m[hh];
        sm_l[warp][hh] = l[hh];
      }
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

}  // namespace wpattn
