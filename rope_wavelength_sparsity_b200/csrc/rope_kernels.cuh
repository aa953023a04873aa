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

// One tensor of a rotation launch: x [B, N, H, D] bf16 turned into out (which
// may be x).  Token t of sequence b sits at pos[b * N + t] when pos is given,
// else at pos0 + t.
struct RopeSegment {
  const uint16_t* x;
  uint16_t* out;
  const int32_t* pos;
  int64_t pos0;
  int64_t N;
  int H;
};

// A launch turns one or two tensors (a prefill's q and k go in one launch, so
// the second does not pay a launch and its ramp of its own).
struct RopeParams {
  RopeSegment seg[2];
  int nseg;
  uint64_t items0;        // (token, chunk) items of seg[0]; seg[1]'s follow
  uint64_t items;         // all items
  double theta[64];       // theta_p = base^(-2p/D)
};

// One thread per (token, chunk of 8 pairs): the eight angles of the chunk are
// turned into cosines and sines once and reused for every head of the token;
// per head two 16-byte loads (dims 8c..8c+7 and D/2+8c..D/2+8c+7) and two
// 16-byte stores.  Heads go four at a time, all four heads' loads issued
// before any of their stores, so that each thread keeps 128 bytes in flight
// instead of waiting a memory round trip per head; the first four heads'
// loads are issued before the angles are computed, so that the trigonometry
// runs under their round trip.  Every element is read before the same thread
// writes it (and a thread's heads are disjoint), so out may alias x.
// Grid-stride over the (token, chunk) items of both tensors.
template <int D>
__global__ void __launch_bounds__(256) rope_kernel(const __grid_constant__ RopeParams p) {
  constexpr int P = D / 2, NC = P / 8, HB = 4;
  for (uint64_t idx = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < p.items;
       idx += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    const bool second = idx >= p.items0;
    const RopeSegment& sg = p.seg[second ? 1 : 0];
    const uint64_t li = second ? idx - p.items0 : idx;
    const int c = static_cast<int>(li % NC);
    const uint64_t token = li / NC;
    const int H = sg.H;
    const uint64_t th0 = token * static_cast<uint64_t>(H);
    // load the two 16-byte chunks of heads h .. h + nb - 1
    uint4 lo[HB], hi[HB];
    auto load_batch = [&](int h, int nb) {
#pragma unroll
      for (int u = 0; u < HB; ++u) {
        if (u < nb) {
          const uint16_t* row = sg.x + (th0 + h + u) * D;
          lo[u] = *reinterpret_cast<const uint4*>(row + 8 * c);
          hi[u] = *reinterpret_cast<const uint4*>(row + P + 8 * c);
        }
      }
    };
    int nb = H < HB ? H : HB;
    load_batch(0, nb);
    const int64_t pos = sg.pos ? static_cast<int64_t>(sg.pos[token])
                               : sg.pos0 + static_cast<int64_t>(token % static_cast<uint64_t>(sg.N));
    float cs[8], sn[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) rope_cos_sin(pos, p.theta[8 * c + e], cs[e], sn[e]);
    // rotate one head's two 16-byte chunks and store them
    auto rotate_store = [&](uint64_t th, const uint4& l, const uint4& h2) {
      const uint32_t a[4] = {l.x, l.y, l.z, l.w};
      const uint32_t b[4] = {h2.x, h2.y, h2.z, h2.w};
      uint32_t ra[4], rb[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float y0, y1, z0, z1;
        rope_pair_bf16(bf16lo_to_f32(a[k]), bf16lo_to_f32(b[k]), cs[2 * k], sn[2 * k], y0, z0);
        rope_pair_bf16(bf16hi_to_f32(a[k]), bf16hi_to_f32(b[k]), cs[2 * k + 1], sn[2 * k + 1], y1, z1);
        ra[k] = pack_bf16x2(y0, y1);
        rb[k] = pack_bf16x2(z0, z1);
      }
      uint16_t* orow = sg.out + th * D;
      *reinterpret_cast<uint4*>(orow + 8 * c) = make_uint4(ra[0], ra[1], ra[2], ra[3]);
      *reinterpret_cast<uint4*>(orow + P + 8 * c) = make_uint4(rb[0], rb[1], rb[2], rb[3]);
    };
    for (int h = 0;;) {
#pragma unroll
      for (int u = 0; u < HB; ++u)
        if (u < nb) rotate_store(th0 + h + u, lo[u], hi[u]);
      h += nb;
      if (h >= H) break;
      nb = H - h < HB ? H - h : HB;
      load_batch(h, nb);
    }
  }
}

}  // namespace wpattn
