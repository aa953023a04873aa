"""The benchmark's work accounting against brute-force enumeration (CPU).

Every throughput the benchmark reports divides a work count by a device time:
effective FLOPs of a prefill (4 per kept query-key pair-term, the QK product of
two dims, plus 2 D per causal query-key pair for P V), the same under a block
mask, and the algorithmic bytes of a decode (4 bytes per kept K pair of each
key, all of V, the query, the output and the LSE).  Here each count is
enumerated term by term on small shapes, with the oracle's own thresholds
(pair p kept at distance d iff d <= T_p), and compared exactly with the
closed-form counts the benchmark uses.
"""
import math

import numpy as np
import pytest

import bench
import oracle
import rope_wavelength_sparsity_b200 as wp
from rope_wavelength_sparsity_b200.inputs import Workload


def _kept_pairs(T, d):
    """Kept pairs of every distance in d (T nondecreasing): #{p : d <= T_p}."""
    d = np.asarray(d, dtype=np.int64)
    return len(T) - np.searchsorted(T, d, side="left")


def _row_terms(T, i, k_pos0, Nk):
    """(kept pair-terms, causal keys) of the query at position i."""
    kp = k_pos0 + np.arange(Nk, dtype=np.int64)
    d = i - kp
    d = d[d >= 0]
    return int(_kept_pairs(T, d).sum()), int(d.size)


def _brute_prefill_flops(w):
    T, _ = oracle.thresholds(w.D, w.base, w.alpha, w.g)
    eff = off = 0
    for t in range(w.Nq):
        kept, causal = _row_terms(T, w.q_pos0 + t, w.k_pos0, w.Nk)
        eff += 4 * kept + 2 * w.D * causal
        off += 4 * w.D * causal
    return w.B * w.Hq * eff, w.B * w.Hq * off


CASES = [
    Workload("acc-a", "prefill", 1, 2, 1, 64, 300, 300, 1e4, 1.0, 1),
    Workload("acc-b", "prefill", 2, 4, 2, 128, 200, 520, 5e5, 2.0, 8, q_pos0=320),
    Workload("acc-c", "prefill", 1, 3, 3, 64, 130, 130, 10.0, 0.3, 1),
    Workload("acc-d", "prefill", 1, 1, 1, 64, 97, 97, 1e4, math.inf, 8),
    Workload("acc-e", "prefill", 1, 2, 2, 64, 150, 260, 1e4, 1.0, 1, q_pos0=100, k_pos0=-10),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_prefill_flops_equal_enumeration(w):
    win = wp.Window(w.D, w.base, w.alpha, w.g)
    assert bench.prefill_flops(w, win, wp) == _brute_prefill_flops(w)


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_oracle_row_flops_sum_to_the_prefill(w):
    """The oracle arm's per-row count (the oracle's own pair-term count) against the
    enumeration, and summed over every row against the product's closed form."""
    win = wp.Window(w.D, w.base, w.alpha, w.g)
    T, _ = oracle.thresholds(w.D, w.base, w.alpha, w.g)
    rows = [0, w.Nq // 2, w.Nq - 1]
    for t in rows:
        kept, causal = _row_terms(T, w.q_pos0 + t, w.k_pos0, w.Nk)
        assert bench.row_flops_oracle(w, t) == 4 * kept + 2 * w.D * causal
    total = sum(bench.row_flops_oracle(w, t) for t in range(w.Nq))
    assert w.B * w.Hq * total == bench.prefill_flops(w, win, wp)[0]


@pytest.mark.parametrize("g,alpha", [(1, 1.0), (8, 1.0), (1, math.inf)])
def test_oracle_decode_row_bytes(g, alpha):
    """A decode row's share of its group's K slice and V, by the oracle's count, against
    the enumeration; G rows of one (sequence, kv head) add up to the group's bytes."""
    w = Workload("acc-dec-row", "decode", 2, 6, 2, 128, 1, 700, 5e5, alpha, g)
    T, _ = oracle.thresholds(w.D, w.base, w.alpha, w.g)
    G = w.Hq // w.Hkv
    for L in (1, 257, 700):
        d = (L - 1) - np.arange(L, dtype=np.int64)
        kept = int(_kept_pairs(T, d).sum())
        assert bench.decode_row_bytes_oracle(w, L) * G == pytest.approx(4 * kept + 2 * w.D * L)


@pytest.mark.parametrize("g,alpha", [(1, 1.0), (8, 1.0), (1, math.inf), (8, 0.05)])
def test_decode_bytes_equal_enumeration(g, alpha):
    w = Workload("acc-dec", "decode", 3, 6, 2, 128, 1, 700, 5e5, alpha, g)
    kv_len = [700, 1, 257]
    win = wp.Window(w.D, w.base, w.alpha, w.g)
    T, _ = oracle.thresholds(w.D, w.base, w.alpha, w.g)
    alg = full = 0
    for L in kv_len:
        d = (L - 1) - np.arange(L, dtype=np.int64)   # distances of keys 0 .. L-1
        kept = int(_kept_pairs(T, d).sum())
        alg += w.Hkv * (4 * kept + 2 * w.D * L)        # kept K pairs, 2 dims x 2 bytes; all of V
        full += w.Hkv * (4 * (w.D // 2) * L + 2 * w.D * L)
    io = w.B * w.Hq * (2 * w.D * 2 + 4)                # query and output bf16, LSE fp32
    assert bench.decode_bytes(w, win, wp, kv_len) == (alg + io, full + io)


def test_masked_flops_equal_enumeration():
    import torch
    w = Workload("acc-mask", "prefill", 1, 2, 1, 64, 300, 300, 1e4, 1.0, 1)
    blk = wp.MASK_BLOCK
    nqb = (w.Nq + blk - 1) // blk
    nkb = (w.Nk + blk - 1) // blk
    rng = np.random.default_rng(3)
    mask = torch.from_numpy(rng.random((w.B, w.Hq, nqb, nkb)) < 0.6)
    win = wp.Window(w.D, w.base, w.alpha, w.g)
    T, _ = oracle.thresholds(w.D, w.base, w.alpha, w.g)
    want = 0
    for b, h, qb, kb in mask.nonzero().tolist():
        for t in range(qb * blk, min(w.Nq, (qb + 1) * blk)):
            k0 = kb * blk
            nk = min(w.Nk, k0 + blk) - k0
            kept, causal = _row_terms(T, w.q_pos0 + t, w.k_pos0 + k0, nk)
            want += 4 * kept + 2 * w.D * causal
    assert bench.masked_flops(w, win, wp, mask) == want
    # every block attended: the unmasked count
    ones = torch.ones((w.B, w.Hq, nqb, nkb), dtype=torch.bool)
    assert bench.masked_flops(w, win, wp, ones) == bench.prefill_flops(w, win, wp)[0]


def test_kernel_hash_ignores_comments_not_code():
    """The traffic table's key: a comment or layout change keeps the hash, a code change
    does not."""
    import bench
    a = "int f(int x) {  // twice\n  return 2 * x; /* doubled */\n}\n"
    b = "// the same function\nint f(int x) {\n    return 2 * x;\n}"
    c = "int f(int x) { return 3 * x; }"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
    assert len(bench.kernel_source_hash("prefill")) == 16
