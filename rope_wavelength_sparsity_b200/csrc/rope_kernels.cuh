// RoPE application for inputs that arrive before their rotation.
//
// WavePrune, Original abstract: RoPE turns each 2-D channel of a query or key
// at a channel-specific frequency.  Pair p = dims (p, p + D/2) turns by
// pos * theta_p, theta_p = base^(-2p/D) (wavelength 2 pi base^(2p/D), the
// form of "The Heterogeneous Feature of RoPE-based Attention", Length
// Extrapolation formula).  The rotated values are rounded to bf16, as a model
// that stores its rotated queries and keys in bf16 would hold them; the
// window and the attention then run on those values unchanged.
#pragma once

#include <cstdint>

#include "device_util.cuh"

namespace wpattn {

constexpr double kTwoPiD = 6.283185307179586476925286766559;

// cos and sin of pos * theta: the angle is reduced modulo 2 pi in double
// precision (positions reach 2^31, where a float angle would be off by whole
// radians), then sincosf runs on the remainder, |r| <= pi.
__device__ __forceinline__ void rope_cos_sin(int64_t pos, double theta, float& c, float& s) {
  const double a = static_cast<double>(pos) * theta;
  const double k = rint(a * (1.0 / kTwoPiD));
  const float r = static_cast<float>(fma(-k, kTwoPiD, a));
  sincosf(r, &s, &c);
}

// One rotated pair, each value rounded to bf16 (returned as its float value).
__device__ __forceinline__ void rope_pair_bf16(float x0, float x1, float c, float s, float& y0,
                                               float& y1) {
  const float r0 = fmaf(x0, c, -(x1 * s));
  const float r1 = fmaf(x0, s, x1 * c);
  y0 = __uint_as_float((pack_bf16x2(r0, 0.f) & 0xFFFFu) << 16);
  y1 = __uint_as_float((pack_bf16x2(r1, 0.f) & 0xFFFFu) << 16);
}

struct RopeParams {
  const uint16_t* x;      // [B, N, H, D] bf16
  uint16_t* out;          // [B, N, H, D] bf16 (may be x)
  const int32_t* pos;     // [B, N] positions, or null: token t of every sequence at pos0 + t
  int64_t pos0;
  int64_t B, N;
  int H;
  double theta[64];       // theta_p = base^(-2p/D)
};

// One thread per (token, chunk of 8 pairs): the eight angles of the chunk are
// turned into cosines and sines once and reused for every head of the token;
// per head two 16-byte loads (dims 8c..8c+7 and D/2+8c..D/2+8c+7) and two
// 16-byte stores.  Heads go four at a time, all four heads' loads issued
// before any of their stores, so that each thread keeps 128 bytes in flight
// instead of waiting a memory round trip per head.  Every element is read
// before the same thread writes it (and a thread's heads are disjoint), so
// out may alias x.  Grid-stride over the (token, chunk) items.
template <int D>
__global__ void __launch_bounds__(256) rope_kernel(const __grid_constant__ RopeParams p) {
  constexpr int P = D / 2, NC = P / 8, HB = 4;
  const uint64_t n = static_cast<uint64_t>(p.B) * p.N * NC;
  for (uint64_t idx = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < n;
       idx += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx % NC);
    const uint64_t token = idx / NC;
    const int64_t pos = p.pos ? static_cast<int64_t>(p.pos[token])
                              : p.pos0 + static_cast<int64_t>(token % static_cast<uint64_t>(p.N));
    float cs[8], sn[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) rope_cos_sin(pos, p.theta[8 * c + e], cs[e], sn[e]);
    // rotate one head's two 16-byte chunks and store them
    auto rotate_store = [&](uint64_t th, const uint4& lo, const uint4& hi) {
      const uint32_t a[4] = {lo.x, lo.y, lo.z, lo.w};
      const uint32_t b[4] = {hi.x, hi.y, hi.z, hi.w};
      uint32_t ra[4], rb[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float y0, y1, z0, z1;
        rope_pair_bf16(bf16lo_to_f32(a[k]), bf16lo_to_f32(b[k]), cs[2 * k], sn[2 * k], y0, z0);
        rope_pair_bf16(bf16hi_to_f32(a[k]), bf16hi_to_f32(b[k]), cs[2 * k + 1], sn[2 * k + 1], y1, z1);
        ra[k] = pack_bf16x2(y0, y1);
        rb[k] = pack_bf16x2(z0, z1);
      }
      uint16_t* orow = p.out + th * D;
      *reinterpret_cast<uint4*>(orow + 8 * c) = make_uint4(ra[0], ra[1], ra[2], ra[3]);
      *reinterpret_cast<uint4*>(orow + P + 8 * c) = make_uint4(rb[0], rb[1], rb[2], rb[3]);
    };
    const uint64_t th0 = token * static_cast<uint64_t>(p.H);
    int h = 0;
    for (; h + HB <= p.H; h += HB) {
      uint4 lo[HB], hi[HB];
#pragma unroll
      for (int u = 0; u < HB; ++u) {
        const uint16_t* row = p.x + (th0 + h + u) * D;
        lo[u] = *reinterpret_cast<const uint4*>(row + 8 * c);
        hi[u] = *reinterpret_cast<const uint4*>(row + P + 8 * c);
      }
#pragma unroll
      for (int u = 0; u < HB; ++u) rotate_store(th0 + h + u, lo[u], hi[u]);
    }
    for (; h < p.H; ++h) {
      const uint16_t* row = p.x + (th0 + h) * D;
      const uint4 lo = *reinterpret_cast<const uint4*>(row + 8 * c);
      const uint4 hi = *reinterpret_cast<const uint4*>(row + P + 8 * c);
      rotate_store(th0 + h, lo, hi);
    }
  }
}

}  // namespace wpattn
