// Host-side planner for windowed attention: per-pair thresholds, the
// closed-form pruned-term count and the decode split plan.  All device
// kernels compare integers against the thresholds computed here, so the
// window the kernels apply is exactly the one this file defines.
#pragma once

#include <cstddef>
#include <cstdint>

#include "wpattn.h"

namespace wpattn {

constexpr int kMaxPairs = 64;                 // D <= 128 on the GPU paths
constexpr int64_t kNoLimit = INT64_MAX;       // threshold of a disabled window

struct WindowPlan {
  int D = 0;        // head dim
  int P = 0;        // pairs = D / 2
  int g = 1;        // pair granularity
  bool off = false; // alpha = +inf
  int64_t T[kMaxPairs];  // per-pair threshold (group value when g = 8), nondecreasing
};

// Validates the window and fills `plan`.  Returns a WPATTN_* code; a head
// dim above 2 * kMaxPairs (D > 128) gives WPATTN_EUNSUPPORTED, and such
// windows are only evaluated on the host, pair by pair, through
// pair_threshold / effective_threshold (the thresholds and the pruned count).
int make_window_plan(const wpattn_window* w, WindowPlan* plan);

// Threshold of pair p for arbitrary even D (host count path for D > 128).
int64_t pair_threshold(const wpattn_window* w, int p);
int64_t effective_threshold(const wpattn_window* w, int p);

// Number of pairs pruned at distance d: #{p : T_p < d}.  The kept set is the
// suffix p >= p_min(d) because thresholds grow with p.
inline int p_min(const WindowPlan& plan, int64_t d) {
  int lo = 0, hi = plan.P;  // first index with T >= d
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (plan.T[mid] < d) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Kept terms of one pair with threshold T summed over the rows of a prefill
// (closed form, O(1)); rows u = q_pos0 - k_pos0 + t, t < Nq; keys 0..Nk-1.
unsigned __int128 kept_terms_one_pair(int64_t T, int64_t Nq, int64_t Nk, int64_t q_pos0,
                                      int64_t k_pos0);

// Decode split plan: every sequence is cut into `splits` key ranges of
// `chunk(kv_len)` keys (a multiple of 64).
struct DecodeSplit {
  int splits = 1;
  int max_splits = 1;  // what the workspace was sized for
};

int decode_max_splits(int B, int Hkv, int64_t max_kv_len);
// Splits per (sequence, kv head) for a GPU that holds `slots` decode CTAs at
// once (SMs x resident CTAs per SM): at most one wave, since a partial second
// wave of CTAs that stream the same number of bytes runs at a fraction of the
// bandwidth and leaves the first wave's SMs idle.
int decode_splits(int B, int Hkv, int64_t max_kv_len, int slots);
size_t decode_workspace_bytes(int B, int Hq, int D, int max_splits);

}  // namespace wpattn
