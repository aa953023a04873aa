// Host planner: thresholds, closed-form pruned-term count, decode split plan.
//
// Window definition ("ATFlash: Per-RoPE-Wavelength Attention Windows",
// Abstract; "WavePrune", Original abstract): pair p (dims p, p + D/2) has
// wavelength lambda_p = 2*pi*base^(2p/D) and keeps its term while the
// query-key distance is at most T_p = floor(alpha * lambda_p).  With g = 8
// pairs share the threshold of their group's longest wavelength.
#include "planner.h"

#include <cmath>

namespace wpattn {

namespace {
constexpr double kTwoPi = 6.28318530717958647692528676655900577;  // nearest double to 2*pi

bool window_fields_ok(const wpattn_window* w) {
  if (!w) return false;
  if (w->head_dim <= 0 || (w->head_dim & 1)) return false;
  if (!(w->rope_base > 1.0) || std::isinf(w->rope_base)) return false;
  if (!(w->alpha > 0.0)) return false;  // rejects NaN and <= 0
  if (w->group_pairs != 1 && w->group_pairs != 8) return false;
  if (w->group_pairs == 8 && ((w->head_dim / 2) % 8) != 0) return false;
  return true;
}
}  // namespace

int64_t pair_threshold(const wpattn_window* w, int p) {
  if (std::isinf(w->alpha)) return kNoLimit;
  const double lam = kTwoPi * std::pow(w->rope_base, static_cast<double>(2 * p) /
                                                         static_cast<double>(w->head_dim));
  const double reach = w->alpha * lam;
  if (!(reach < 4.0e18)) return kNoLimit;
  return static_cast<int64_t>(std::floor(reach));
}

int64_t effective_threshold(const wpattn_window* w, int p) {
  if (w->group_pairs == 1) return pair_threshold(w, p);
  // lambda grows with p, so the group's longest wavelength is its last pair
  return pair_threshold(w, (p / 8) * 8 + 7);
}

int make_window_plan(const wpattn_window* w, WindowPlan* plan) {
  if (!window_fields_ok(w)) return WPATTN_EINVAL;
  if (w->head_dim / 2 > kMaxPairs) return WPATTN_EUNSUPPORTED;
  plan->D = w->head_dim;
  plan->P = w->head_dim / 2;
  plan->g = w->group_pairs;
  plan->off = std::isinf(w->alpha);
  for (int p = 0; p < plan->P; ++p) plan->T[p] = effective_threshold(w, p);
  for (int p = plan->P; p < kMaxPairs; ++p) plan->T[p] = kNoLimit;
  return WPATTN_OK;
}

namespace {
using u128 = unsigned __int128;

// Sum_{u=0}^{x} f(u) where, for u >= 0, f(u) = max(0, 1 + min(u, T, L, T + L - u)):
// the number of kept distances of a query row u steps after the first key,
// with keys at distances [max(0, u - L), u] and pair threshold T.
// f rises as u+1 up to A = min(T, L), stays A+1 up to Bv = max(T, L), then
// falls as T+L-u+1 to 0 at u = T+L+1.
u128 trapezoid_prefix(int64_t x, int64_t T, int64_t L) {
  if (x < 0) return 0;
  const int64_t A = T < L ? T : L;
  const int64_t Bv = T < L ? L : T;
  const int64_t E = T + L;
  u128 s = 0;
  const int64_t n1 = (x < A ? x : A) + 1;
  s += static_cast<u128>(n1) * static_cast<u128>(n1 + 1) / 2;
  const int64_t hi2 = x < Bv ? x : Bv;
  if (hi2 > A) s += static_cast<u128>(A + 1) * static_cast<u128>(hi2 - A);
  const int64_t lo3 = Bv + 1;
  const int64_t hi3 = x < E ? x : E;
  if (hi3 >= lo3) {
    const u128 first = static_cast<u128>(A);              // value at u = lo3
    const u128 last = static_cast<u128>(E - hi3 + 1);     // value at u = hi3
    s += (first + last) * static_cast<u128>(hi3 - lo3 + 1) / 2;
  }
  return s;
}
}  // namespace

u128 kept_terms_one_pair(int64_t T, int64_t Nq, int64_t Nk, int64_t q_pos0, int64_t k_pos0) {
  if (Nq <= 0 || Nk <= 0) return 0;
  const int64_t u0 = q_pos0 - k_pos0;
  const int64_t u_end = u0 + Nq - 1;
  if (u_end < 0) return 0;
  const int64_t a = u0 > 0 ? u0 : 0;
  const int64_t L = Nk - 1;
  // beyond the last row's distance the threshold no longer matters
  const int64_t Tc = T < u_end ? T : u_end;
  return trapezoid_prefix(u_end, Tc, L) - trapezoid_prefix(a - 1, Tc, L);
}

// ------------------------------------------------------------- decode plan
namespace {
constexpr int kMaxDecodeCtas = 4096;
constexpr int64_t kMinKeysPerSplit = 256;
}  // namespace

int decode_max_splits(int B, int Hkv, int64_t max_kv_len) {
  const int64_t units = static_cast<int64_t>(B) * Hkv;
  int64_t s = (kMaxDecodeCtas + units - 1) / units;
  const int64_t by_len = (max_kv_len + kMinKeysPerSplit - 1) / kMinKeysPerSplit;
  if (s > by_len) s = by_len;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

int decode_splits(int B, int Hkv, int64_t max_kv_len, int slots) {
  const int64_t units = static_cast<int64_t>(B) * Hkv;
  const int64_t target = slots > 0 ? slots : 148 * 3;
  int64_t s = target / units;
  const int smax = decode_max_splits(B, Hkv, max_kv_len);
  if (s > smax) s = smax;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

size_t decode_workspace_bytes(int B, int Hq, int D, int max_splits) {
  const size_t rec = static_cast<size_t>(D + 2) * sizeof(float);
  const size_t bytes = static_cast<size_t>(B) * Hq * max_splits * rec;
  return (bytes + 255) / 256 * 256;
}

}  // namespace wpattn
