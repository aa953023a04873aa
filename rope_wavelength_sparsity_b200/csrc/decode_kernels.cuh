// Split-KV decode for windowed attention (one new query per sequence).
//
// "ATFlash: Per-RoPE-Wavelength Attention Windows", Abstract: the window is
// a slice of the query-key contraction axis ported into a FlashInfer-style
// decode kernel.  Here every key's K row is read only over the 16-byte
// chunks (8 head dims) that still hold a kept pair at that key's distance;
// V rows are read in full.  A warp holds 32/(D/8) keys per load step, one
// 16-byte chunk per lane, so K and V loads are coalesced 16-byte vectors;
// the per-key dot product is a shuffle reduction across the D/8 lanes of
// the key.  Each CTA covers one (sequence, kv head, key range) and all the
// query heads of the GQA group (up to GC at a time), so a K/V byte is read
// once for the group.  A second kernel merges the key ranges by their
// log-sum-exp.
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

__host__ __device__ constexpr int decode_keys_per_cta_step(int D) {
  return (kDecodeThreads / 32) * (32 / (D / 8));
}

template <int D, int GC>
__global__ void __launch_bounds__(kDecodeThreads)
decode_split_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int TPK = D / 8;              // lanes per key (one 16-byte chunk each)
  constexpr int KPW = 32 / TPK;           // keys per warp per load step
  constexpr int KPC = (kDecodeThreads / 32) * KPW;  // keys per CTA per load step
  constexpr int U = 4;                    // load steps in flight per iteration
  constexpr int HALF = TPK / 2;           // chunks per half of the head dim

  __shared__ float sm_m[KPC][GC];
  __shared__ float sm_l[KPC][GC];
  __shared__ float sm_o[KPC][GC][D];

  const int split = blockIdx.x;
  const int kvh = blockIdx.y / p.hchunks;
  const int hc = blockIdx.y % p.hchunks;
  const int b = blockIdx.z;
  const int h0 = kvh * p.G + hc * GC;
  const int nh = min(GC, p.G - hc * GC);
  const int L = p.kv_len[b];
  const int chunk = ((L + p.S - 1) / p.S + 63) / 64 * 64;
  const int j_begin = split * chunk;
  const int j_end = min(L, j_begin + chunk);
  const int qpos = L - 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = lane % TPK;               // head-dim chunk [8c, 8c+8)
  const int slot = warp * KPW + lane / TPK;
  const int pb = (c % HALF) * 8;          // first pair of this chunk
  int Tc[8];  // thresholds of this chunk's 8 pairs
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

  const size_t row_stride = (size_t)p.Hkv * D;
  const uint16_t* kbase = p.k + ((size_t)b * p.Lmax * p.Hkv + kvh) * D + 8 * c;
  const uint16_t* vbase = p.v + ((size_t)b * p.Lmax * p.Hkv + kvh) * D + 8 * c;

  for (int jb = j_begin; jb < j_end; jb += KPC * U) {
    uint4 kraw[U], vraw[U];
    int dist[U];
    bool valid[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = jb + u * KPC + slot;
      valid[u] = j < j_end;
      dist[u] = qpos - j;
      const bool kact = valid[u] && dist[u] <= T_last;  // chunk holds a kept pair
      kraw[u] = kact ? ldg_stream(kbase + (size_t)j * row_stride) : make_uint4(0, 0, 0, 0);
      vraw[u] = valid[u] ? ldg_stream(vbase + (size_t)j * row_stride) : make_uint4(0, 0, 0, 0);
    }
    float s[U][GC];
    float vf[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      unpack8(vraw[u], vf[u]);
      float kf[8];
      unpack8(kraw[u], kf);
      if (dist[u] > T_first) {  // chunk only partly kept at this distance
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (dist[u] > Tc[e]) kf[e] = 0.f;
      }
#pragma unroll
      for (int hh = 0; hh < GC; ++hh) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc = fmaf(qf[hh][e], kf[e], acc);
#pragma unroll
        for (int off = TPK / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        s[u][hh] = valid[u] ? acc : -INFINITY;
      }
    }
#pragma unroll
    for (int hh = 0; hh < GC; ++hh) {
      float mx = m[hh];
#pragma unroll
      for (int u = 0; u < U; ++u) mx = fmaxf(mx, s[u][hh]);
      if (mx == -INFINITY) continue;
      const float corr = ex2_approx(m[hh] - mx);
      l[hh] *= corr;
#pragma unroll
      for (int e = 0; e < 8; ++e) o[hh][e] *= corr;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float pu = ex2_approx(s[u][hh] - mx);
        l[hh] += pu;
#pragma unroll
        for (int e = 0; e < 8; ++e) o[hh][e] = fmaf(pu, vf[u][e], o[hh][e]);
      }
      m[hh] = mx;
    }
  }

  // merge the KPC key slots of this CTA
#pragma unroll
  for (int hh = 0; hh < GC; ++hh) {
#pragma unroll
    for (int e = 0; e < 8; ++e) sm_o[slot][hh][8 * c + e] = o[hh][e];
    if (c == 0) {
      sm_m[slot][hh] = m[hh];
      sm_l[slot][hh] = l[hh];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < nh * D; idx += kDecodeThreads) {
    const int hh = idx / D, e = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int s2 = 0; s2 < KPC; ++s2) M = fmaxf(M, sm_m[s2][hh]);
    float Ls = 0.f, Os = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int s2 = 0; s2 < KPC; ++s2) {
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
