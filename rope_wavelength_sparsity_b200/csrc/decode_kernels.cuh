// Split-KV decode for windowed attention (one new query per sequence).
//
// "ATFlash: Per-RoPE-Wavelength Attention Windows", Abstract: the window is
// a slice of the query-key contraction axis ported into a FlashInfer-style
// decode kernel.  Each CTA covers one (sequence, kv head, key range) and all
// the query heads of the GQA group (up to GC at a time), so a K/V byte is
// read once for the group.  A producer warp streams blocks of 32 keys of K
// and V through a shared-memory ring with TMA (128-byte swizzle); four
// compute warps take one 16-byte chunk (8 head dims) of a key per lane, so
// a warp holds 32/(D/8) keys per step.  A lane multiplies its K chunk only
// if the chunk still holds a kept pair at that key's distance (pruned dims
// are zeroed); the dot product is a shuffle reduction across the key's lanes.
// In the [B, L, Hkv, D] cache layout each half of a K row is one 128-byte
// line and the kept slice touches both, so whole rows move from DRAM either
// way; the window saves arithmetic here, not bytes.  A second kernel merges
// the key ranges by their log-sum-exp.
#pragma once

#include "device_util.cuh"

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
  int kv_len[kDecodeMaxB];
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
// the 128-byte-swizzled layout TMA writes (64-dim panels, row = key).
template <int D>
struct DecodeSmem {
  static constexpr int KB = 32;                        // keys per block
  static constexpr int NS = (D == 64) ? 8 : 4;         // ring depth
  static constexpr int PANEL = KB * 128;               // one 64-dim panel of a block
  static constexpr int TILE = KB * D * 2;              // K or V block
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = NS * TILE;
  static constexpr int OFF_BAR = 2 * NS * TILE;        // full[NS], empty[NS]
  static constexpr int BYTES = OFF_BAR + 2 * NS * 8;
  static constexpr int ALLOC = BYTES + 1024;           // slack to align the ring to 1024 bytes
};

// compute warps per CTA: more warps (and fewer live values each) for large
// GQA groups, whose per-lane accumulators limit occupancy
__host__ __device__ constexpr int decode_compute_warps(int GC) { return GC > 4 ? 8 : 4; }

// 16 bytes of a K or V row from the swizzled ring: row r (key within the
// block), 16-byte chunk c of the head dim.
template <int D>
__device__ __forceinline__ uint4 ring_chunk(const uint8_t* tile, int r, int c) {
  using L = DecodeSmem<D>;
  return *reinterpret_cast<const uint4*>(tile + (c >> 3) * L::PANEL + r * 128 +
                                         (((c & 7) ^ (r & 7)) << 4));
}

template <int D, int GC>
__global__ void __launch_bounds__((decode_compute_warps(GC) + 1) * 32)
decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ DecodeParams p) {
  using L = DecodeSmem<D>;
  constexpr int KB = L::KB, NS = L::NS;
  constexpr int kDecodeComputeWarps = decode_compute_warps(GC);
  constexpr int TPK = D / 8;              // lanes per key (one 16-byte chunk each)
  constexpr int KPW = 32 / TPK;           // keys per warp per step
  constexpr int SLOTS = kDecodeComputeWarps * KPW;
  constexpr int U = KB / SLOTS;           // steps per block
  constexpr int HALF = TPK / 2;           // chunks per half of the head dim
  static_assert(KB % SLOTS == 0, "block must be a multiple of the key slots");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the swizzled ring starts on a 1024-byte boundary of the shared window
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ float sm_m[SLOTS][GC];
  __shared__ float sm_l[SLOTS][GC];
  // the merge's partial outputs reuse the ring once every block is consumed
  static_assert(SLOTS * GC * D * 4 <= 2 * NS * L::TILE, "merge buffer must fit in the ring");
  float (*sm_o)[GC][D] = reinterpret_cast<float (*)[GC][D]>(smem);

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
  const int qpos = Lb - 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), kDecodeComputeWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kDecodeComputeWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      for (int i = 0; i < nblk; ++i) {
        const int s = i % NS;
        if (i >= NS && !mbar_wait(empty(s), ((i / NS) & 1) ^ 1)) break;
        mbar_arrive_expect_tx(full(s), 2 * L::TILE);
        const int j0 = j_begin + i * KB;
        for (int c = 0; c < D / 64; ++c) {
          tma_load_4d(sbase + L::OFF_K + s * L::TILE + c * L::PANEL, &tmK, full(s), 64 * c, j0, kvh, b);
          tma_load_4d(sbase + L::OFF_V + s * L::TILE + c * L::PANEL, &tmV, full(s), 64 * c, j0, kvh, b);
        }
      }
    }
    return;  // the producer takes no part in the merge below
  }

  // ---------------------------------------------------------------- compute
  const int c = lane % TPK;               // head-dim chunk [8c, 8c+8)
  const int slot = warp * KPW + lane / TPK;
  const int pb = (c % HALF) * 8;          // first pair of this chunk
  int Tc[8];                              // thresholds of this chunk's 8 pairs
#pragma unroll
  for (int e = 0; e < 8; ++e) Tc[e] = p.T[pb + e];
  const int T_first = Tc[0];
  const int T_last = Tc[7];

  float qf[GC][8];
#pragma unroll
  for (int hh = 0; hh < GC; ++hh) {
    if (hh < nh) {
      const uint4 u = *reinterpret_cast<const uint4*>(p.q + ((size_t)b * p.Hq + h0 + hh) * D + 8 * c);
      unpack8(u, qf[hh]);
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[hh][e] *= p.scale_log2;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[hh][e] = 0.f;
    }
  }
  float m[GC], l[GC], o[GC][8];
#pragma unroll
  for (int hh = 0; hh < GC; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[hh][e] = 0.f;
  }

  bool ok = true;
  for (int i = 0; i < nblk; ++i) {
    const int s = i % NS;
    if (!__all_sync(0xffffffffu, mbar_wait(full(s), (i / NS) & 1))) { ok = false; break; }
    const uint8_t* kt = smem + L::OFF_K + s * L::TILE;
    const uint8_t* vt = smem + L::OFF_V + s * L::TILE;
    float sco[U][GC];
    float vf[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = u * SLOTS + slot;     // key within the block
      const int j = j_begin + i * KB + r;
      const bool valid = j < j_end;
      const int dist = qpos - j;
      unpack8(ring_chunk<D>(vt, r, c), vf[u]);
      float kf[8];
      if (dist <= T_last) {               // this chunk holds a kept pair
        unpack8(ring_chunk<D>(kt, r, c), kf);
        if (dist > T_first) {             // only partly kept at this distance
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (dist > Tc[e]) kf[e] = 0.f;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) kf[e] = 0.f;
      }
#pragma unroll
      for (int hh = 0; hh < GC; ++hh) {
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int e = 0; e < 8; e += 2)
          fma2(a0, a1, qf[hh][e], qf[hh][e + 1], kf[e], kf[e + 1], a0, a1);
        float acc = a0 + a1;
#pragma unroll
        for (int off = TPK / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        sco[u][hh] = valid ? acc : -INFINITY;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(s));
#pragma unroll
    for (int hh = 0; hh < GC; ++hh) {
      float mx = m[hh];
#pragma unroll
      for (int u = 0; u < U; ++u) mx = fmaxf(mx, sco[u][hh]);
      if (mx == -INFINITY) continue;
      const float corr = ex2_approx(m[hh] - mx);
      l[hh] *= corr;
#pragma unroll
      for (int e = 0; e < 8; e += 2) mul2(o[hh][e], o[hh][e + 1], o[hh][e], o[hh][e + 1], corr, corr);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float pu = ex2_approx(sco[u][hh] - mx);
        l[hh] += pu;
#pragma unroll
        for (int e = 0; e < 8; e += 2)
          fma2(o[hh][e], o[hh][e + 1], pu, pu, vf[u][e], vf[u][e + 1], o[hh][e], o[hh][e + 1]);
      }
      m[hh] = mx;
    }
  }
  (void)ok;

  // merge the key slots of this CTA (compute warps only); every block has
  // been consumed, so the ring is free
  asm volatile("bar.sync 1, %0;" ::"n"(kDecodeComputeWarps * 32) : "memory");
#pragma unroll
  for (int hh = 0; hh < GC; ++hh) {
#pragma unroll
    for (int e = 0; e < 8; ++e) sm_o[slot][hh][8 * c + e] = o[hh][e];
    if (c == 0) {
      sm_m[slot][hh] = m[hh];
      sm_l[slot][hh] = l[hh];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kDecodeComputeWarps * 32) : "memory");
  for (int idx = threadIdx.x; idx < nh * D; idx += kDecodeComputeWarps * 32) {
    const int hh = idx / D, e = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int s2 = 0; s2 < SLOTS; ++s2) M = fmaxf(M, sm_m[s2][hh]);
    float Ls = 0.f, Os = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int s2 = 0; s2 < SLOTS; ++s2) {
        const float w = ex2_approx(sm_m[s2][hh] - M);
        Ls += sm_l[s2][hh] * w;
        Os += sm_o[s2][hh][e] * w;
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
