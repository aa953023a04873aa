"""Write workload_counts.json: the exact pruned pair-term counts of the
benchmark workloads, from the window's definition alone.

ATFlash, Abstract: the pruned share of the query-key pair-terms is
input-independent and has a closed form.  This script evaluates that form
with its own code (it imports nothing from the oracle or the library), so the
stored numbers are an independent check of ``oracle.count_rows``:

* T_p = floor(alpha * 2 pi * base^(2p/D)) for pair p (half-split pairs), the
  group's largest for g = 8 (a group of 8 pairs stays while any member would);
* a query at relative position u = q_pos - k_pos0 sees the distances
  max(0, u - L) .. u, with L = Nk - 1, and pair p keeps those <= T_p;
* per pair, the kept count summed over the rows is a sum of arithmetic series
  over the four regions of u (below both T and L, between them, above both),
  not a loop over rows.

Run from the repository root:  python tests/golden/make_workload_counts.py
"""
import json
import math
import os

T_INF = None  # no limit (alpha = inf)

WORKLOADS = [
    # name, D, base, alpha, g, Nq, Nk, q_pos0, k_pos0, (decode: one row at Nk - 1)
    ("tiny", 64, 1e4, 1.0, 1, 256, 256, 0, 0),
    ("qwen2.5-0.5b-32k", 64, 1e6, 1.0, 8, 32768, 32768, 0, 0),
    ("llama3.2-3b-128k-a1", 128, 5e5, 1.0, 1, 131072, 131072, 0, 0),
    ("llama3.2-3b-128k-a2", 128, 5e5, 2.0, 1, 131072, 131072, 0, 0),
    ("qwen2.5-7b-1m-prefill", 128, 1e7, 1.0, 8, 16384, 1048576, 1048576 - 16384, 0),
    ("llama3.2-3b-decode-128k", 128, 5e5, 1.0, 1, 1, 131072, 131072 - 1, 0),
    ("qwen2.5-7b-1m-decode", 128, 1e7, 1.0, 8, 1, 1048576, 1048576 - 1, 0),
]


def thresholds(D, base, alpha, g):
    P = D // 2
    if math.isinf(alpha):
        return [T_INF] * P
    T = [math.floor(alpha * (2.0 * math.pi * math.pow(base, (2 * p) / D))) for p in range(P)]
    if g == 8:
        T = [T[(p // 8) * 8 + 7] for p in range(P)]
    return T


def _series(a, b, c0, c1):
    """sum_{u=a}^{b} (c0 + c1 * u) for integers a <= b (0 if a > b)."""
    if a > b:
        return 0
    n = b - a + 1
    return c0 * n + c1 * (a + b) * n // 2


def kept_one_pair(T, u0, u1, L):
    """sum over u = u0 .. u1 (u >= 0) of the distances in [max(0, u - L), u] that are <= T."""
    u0 = max(u0, 0)
    if u1 < u0:
        return 0
    if T is None:
        T = u1 + L + 1            # never binds
    lo_TL, hi_TL = min(T, L), max(T, L)
    s = _series(u0, min(u1, lo_TL), 1, 1)                 # u <= min(T, L): u + 1
    if T < L:
        s += _series(max(u0, T + 1), min(u1, L), T + 1, 0)   # T < u <= L: T + 1
    elif L < T:
        s += _series(max(u0, L + 1), min(u1, T), L + 1, 0)   # L < u <= T: L + 1
    top = min(u1, T + L)                                  # u > max(T, L): T + L + 1 - u > 0
    s += _series(max(u0, hi_TL + 1), top, T + L + 1, -1)
    return s


def count(D, base, alpha, g, Nq, Nk, q_pos0, k_pos0):
    """(pruned, total) pair-terms per (batch, head)."""
    L = Nk - 1
    u0, u1 = q_pos0 - k_pos0, q_pos0 - k_pos0 + Nq - 1
    causal = kept_one_pair(None, u0, u1, L)
    P = D // 2
    kept = sum(kept_one_pair(T, u0, u1, L) for T in thresholds(D, base, alpha, g))
    return causal * P - kept, causal * P


def _brute(D, base, alpha, g, Nq, Nk, q_pos0, k_pos0):
    T = thresholds(D, base, alpha, g)
    pr = tot = 0
    for t in range(Nq):
        for j in range(Nk):
            d = (q_pos0 + t) - (k_pos0 + j)
            if d < 0:
                continue
            for Tp in T:
                tot += 1
                pr += 0 if (Tp is None or d <= Tp) else 1
    return pr, tot


def main():
    # the closed form against enumeration on small shapes first
    for case in [(16, 100.0, 1.0, 1, 40, 40, 0, 0), (16, 10.0, 0.3, 8, 30, 70, 25, 0),
                 (8, 50.0, 2.0, 1, 20, 9, 30, 4), (16, 100.0, math.inf, 8, 12, 30, 5, 9)]:
        assert count(*case) == _brute(*case), case
    out = {
        "citation": "ATFlash, Abstract (the pruned share of the QK pair-terms is "
                    "input-independent, with a closed form in N); thresholds T_p = floor(alpha * "
                    "2 pi * base^(2p/D)) per WavePrune, Original abstract (alpha = 1: the first "
                    "rotation period) and the heterogeneous-feature page's wavelength formula.  "
                    "Written by tests/golden/make_workload_counts.py (per-pair arithmetic series, "
                    "no oracle or library code).",
        "units": "pair-terms (query, key, pair) per (batch, head), causal pairs only",
        "workloads": [],
    }
    for (name, D, base, alpha, g, Nq, Nk, q0, k0) in WORKLOADS:
        pruned, total = count(D, base, alpha, g, Nq, Nk, q0, k0)
        out["workloads"].append({"name": name, "D": D, "base": base, "alpha": alpha, "g": g,
                                 "Nq": Nq, "Nk": Nk, "q_pos0": q0, "k_pos0": k0,
                                 "pruned": pruned, "total": total,
                                 "fraction": round(pruned / total, 6)})
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "workload_counts.json")
    with open(path, "w") as fh:
        json.dump(out, fh, indent=1)
        fh.write("\n")
    print(path)


if __name__ == "__main__":
    main()
