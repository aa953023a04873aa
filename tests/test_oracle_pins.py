"""Pins for the oracle: checks against facts other than the oracle itself.

Each test names what it pins and where the fact comes from:
hand-worked examples (tests/golden), a library routine the method reduces to
(torch's scaled_dot_product_attention at alpha = inf), brute-force
enumeration, closed forms of special cases, and invariants of the definition.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from rope_wavelength_sparsity_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return inputs.bits(torch.tensor(x, dtype=torch.float32).to(torch.bfloat16))


def _rand(shape, seed):
    return inputs.randn_bf16(shape, seed)


# ---------------------------------------------------------------------------
# hand-worked examples (ATFlash Abstract; WavePrune Original abstract)
# ---------------------------------------------------------------------------

def test_hand_two_pair_thresholds_scores_and_counts():
    g = json.load(open(os.path.join(GOLD, "hand_two_pair.json")))
    T, _ = oracle.thresholds(g["D"], g["base"], g["alpha"], g["g"])
    assert T.tolist() == g["thresholds"]
    q = _bf16_bits(np.array(g["q"]))
    dmax = max(d for d, _ in g["score_by_distance"])
    keys = _bf16_bits(np.tile(np.array(g["k"]), (dmax + 1, 1)))
    # query at position dmax, key j at position j -> distance dmax - j
    s = oracle.scores(q, keys, q_pos=dmax, base=g["base"], alpha=g["alpha"], g=g["g"])
    for d, want in g["score_by_distance"]:
        assert s[dmax - d] == want, (d, s[dmax - d], want)
    for N, pruned, total in g["counts"]:
        assert oracle.count_bruteforce(g["D"], g["base"], g["alpha"], g["g"], N, N) == (pruned, total)
        assert oracle.count_rows(g["D"], g["base"], g["alpha"], g["g"], N, N) == (pruned, total)


def test_threshold_values_by_hand():
    cases = json.load(open(os.path.join(GOLD, "thresholds.json")))["cases"]
    for c in cases:
        T, margin = oracle.thresholds(c["D"], c["base"], c["alpha"], c["g"])
        assert T[: len(c["first"])].tolist() == c["first"], c
        assert margin > 1e-6


def test_two_pair_softmax_by_hand():
    """Query at position 7 over 8 keys (D = 4, base 100, alpha 1, T = (6, 62)).
    Key 0 (d = 7) = (1,1,1,1): pair 0 pruned, s = 2 + 4 = 6.  Key 7 (d = 0) =
    (0.5, 0, 0.25, 1): s = 0.5 + 0.75 + 4 = 5.25.  Keys 1..6 are zero: s = 0.
    With scale 1 the weights are (e^6, 1, ..., 1, e^5.25) / Z."""
    q = _bf16_bits(np.array([1.0, 2.0, 3.0, 4.0]).reshape(1, 1, 1, 4))
    kk = np.zeros((1, 8, 1, 4))
    vv = np.zeros((1, 8, 1, 4))
    kk[0, 0, 0] = [1.0, 1.0, 1.0, 1.0]
    kk[0, 7, 0] = [0.5, 0.0, 0.25, 1.0]
    vv[0, 0, 0] = [1.0, 0.0, 0.0, 0.0]
    vv[0, 7, 0] = [0.0, 1.0, 0.0, 0.0]
    out, lse = oracle.attention_rows(q, _bf16_bits(kk), _bf16_bits(vv), Hq=1, Hkv=1,
                                     q_pos0=7, k_pos0=0, base=100.0, alpha=1.0, g=1,
                                     scale=1.0, rows=[(0, 0, 0)])
    z = math.exp(6.0) + math.exp(5.25) + 6 * math.exp(0.0)
    assert abs(out[0, 0] - math.exp(6.0) / z) < 1e-12
    assert abs(out[0, 1] - math.exp(5.25) / z) < 1e-12
    assert abs(lse[0] - math.log(z)) < 1e-12


# ---------------------------------------------------------------------------
# alpha = inf reduces to ordinary causal attention (a library routine)
# ---------------------------------------------------------------------------

def _sdpa_reference(q, k, v, Hq, Hkv, q_pos0, k_pos0, scale):
    qf = q.double().permute(0, 2, 1, 3)                # B,Hq,Nq,D
    kf = k.double().repeat_interleave(Hq // Hkv, dim=2).permute(0, 2, 1, 3)
    vf = v.double().repeat_interleave(Hq // Hkv, dim=2).permute(0, 2, 1, 3)
    Nq, Nk = q.shape[1], k.shape[1]
    qp = q_pos0 + torch.arange(Nq)
    kp = k_pos0 + torch.arange(Nk)
    mask = kp[None, :] <= qp[:, None]
    out = torch.nn.functional.scaled_dot_product_attention(qf, kf, vf, attn_mask=mask, scale=scale)
    return out.permute(0, 2, 1, 3)


@pytest.mark.parametrize("D,Hq,Hkv,Nq,Nk,q0,k0", [
    (16, 4, 2, 37, 37, 0, 0),
    (64, 3, 1, 20, 45, 25, 0),
    (8, 2, 2, 9, 30, 100, 80),
])
def test_alpha_inf_is_causal_sdpa(D, Hq, Hkv, Nq, Nk, q0, k0):
    q = _rand((2, Nq, Hq, D), 11)
    k = _rand((2, Nk, Hkv, D), 12)
    v = _rand((2, Nk, Hkv, D), 13)
    scale = 1.0 / math.sqrt(D)
    ref = _sdpa_reference(q, k, v, Hq, Hkv, q0, k0, scale)
    rows = [(b, h, t) for b in range(2) for h in range(Hq) for t in range(Nq)
            if q0 + t >= k0]
    out, lse = oracle.attention_rows(inputs.bits(q), inputs.bits(k), inputs.bits(v), Hq=Hq,
                                     Hkv=Hkv, q_pos0=q0, k_pos0=k0, base=1e4,
                                     alpha=float("inf"), g=1, scale=scale, rows=rows)
    for n, (b, h, t) in enumerate(rows):
        np.testing.assert_allclose(out[n], ref[b, t, h].numpy(), rtol=0, atol=1e-10)


# ---------------------------------------------------------------------------
# special cases with a closed form
# ---------------------------------------------------------------------------

def test_small_alpha_keeps_only_distance_zero():
    """alpha * lambda_{P-1} < 1 (the longest wavelength): every T_p = 0, so a
    key j < i scores exactly 0 and the row's softmax is
    (e^{z_ii}, 1, ..., 1) / (e^{z_ii} + i)."""
    D, N = 16, 24
    alpha = 0.9 / (2 * math.pi * 1e4 ** (2 * 7 / 16))
    T, _ = oracle.thresholds(D, 1e4, alpha, 1)
    assert (T == 0).all()
    q = _rand((1, N, 1, D), 21)
    k = _rand((1, N, 1, D), 22)
    v = _rand((1, N, 1, D), 23)
    scale = 0.25
    rows = [(0, 0, t) for t in range(N)]
    out, lse = oracle.attention_rows(inputs.bits(q), inputs.bits(k), inputs.bits(v), Hq=1,
                                     Hkv=1, base=1e4, alpha=alpha, g=1, scale=scale, rows=rows)
    qd, kd, vd = q.double()[0, :, 0], k.double()[0, :, 0], v.double()[0, :, 0]
    for t in range(N):
        zt = scale * float(qd[t] @ kd[t])
        w_self = math.exp(zt)
        want = (w_self * vd[t] + vd[:t].sum(0)) / (w_self + t)
        np.testing.assert_allclose(out[t], want.numpy(), atol=1e-12)
        assert abs(lse[t] - math.log(w_self + t)) < 1e-12


def test_distance_zero_keeps_every_pair():
    """d = 0 keeps all pairs: the diagonal score is the full dot product."""
    for D, base, alpha, g in [(64, 1e4, 1.0, 1), (128, 5e5, 0.01, 1), (64, 1e6, 0.001, 8)]:
        q = _rand((1, D), 31)
        k = _rand((1, D), 32)
        s = oracle.scores(inputs.bits(q)[0], inputs.bits(k), q_pos=5, k_pos0=5, base=base,
                          alpha=alpha, g=g)
        assert abs(s[0] - float(q.double()[0] @ k.double()[0])) < 1e-12


def test_half_split_pairing_not_interleaved():
    """Pair p couples dims p and p + D/2: with only dims (0, D/2) nonzero in
    q and k, the term survives exactly while pair 0 is kept (d <= T_0)."""
    D = 8
    T, _ = oracle.thresholds(D, 100.0, 1.0, 1)
    qv = np.zeros(D); qv[0] = 1.0; qv[D // 2] = 2.0
    kv = np.zeros(D); kv[0] = 3.0; kv[D // 2] = 5.0
    n = int(T[0]) + 3
    keys = _bf16_bits(np.tile(kv, (n, 1)))
    s = oracle.scores(_bf16_bits(qv), keys, q_pos=n - 1, base=100.0, alpha=1.0, g=1)
    for j in range(n):
        d = n - 1 - j
        assert s[j] == (13.0 if d <= T[0] else 0.0)


def test_group_window_uses_longest_wavelength():
    """g = 8: a group stays while its longest-wavelength member would; with a
    single pair active in q (pair 0), the term survives to T_7, not T_0."""
    D = 16
    T1, _ = oracle.thresholds(D, 100.0, 1.0, 1)
    T8, _ = oracle.thresholds(D, 100.0, 1.0, 8)
    assert (T8 == T1[7]).all()
    qv = np.zeros(D); qv[0] = 1.0
    kv = np.zeros(D); kv[0] = 1.0
    d_probe = int(T1[0]) + 1            # pruned with g = 1, kept with g = 8
    keys = _bf16_bits(np.tile(kv, (d_probe + 1, 1)))
    s1 = oracle.scores(_bf16_bits(qv), keys, q_pos=d_probe, base=100.0, alpha=1.0, g=1)
    s8 = oracle.scores(_bf16_bits(qv), keys, q_pos=d_probe, base=100.0, alpha=1.0, g=8)
    assert s1[0] == 0.0 and s8[0] == 1.0


def test_empty_row_has_zero_output_and_minus_inf_lse():
    q = _rand((1, 4, 1, 16), 41)
    k = _rand((1, 4, 1, 16), 42)
    v = _rand((1, 4, 1, 16), 43)
    out, lse = oracle.attention_rows(inputs.bits(q), inputs.bits(k), inputs.bits(v), Hq=1,
                                     Hkv=1, q_pos0=0, k_pos0=10, base=1e4, alpha=1.0, g=1,
                                     scale=0.25, rows=[(0, 0, 3)])
    assert (out == 0).all() and lse[0] == -math.inf


# ---------------------------------------------------------------------------
# the count: brute force, closed form, logarithmic growth
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("D", [4, 8, 16, 64, 128])
@pytest.mark.parametrize("alpha", [0.05, 0.5, 1.0, 2.0, 7.3, float("inf")])
def test_count_rows_equals_bruteforce(D, alpha):
    for g in (1, 8):
        if g == 8 and (D // 2) % 8:
            continue
        for (Nq, Nk, q0, k0) in [(1, 1, 0, 0), (37, 37, 0, 0), (50, 130, 80, 0),
                                 (64, 20, 10, 30), (5, 300, 299, 0), (40, 40, 0, 50)]:
            bf = oracle.count_bruteforce(D, 100.0 if D <= 8 else 1e4, alpha, g, Nq, Nk, q0, k0)
            rw = oracle.count_rows(D, 100.0 if D <= 8 else 1e4, alpha, g, Nq, Nk, q0, k0)
            assert bf == rw, (D, alpha, g, Nq, Nk, q0, k0)


def test_count_rows_equals_workload_counts():
    """The oracle's row-by-row count at the benchmark workloads' full sizes against
    tests/golden/workload_counts.json, exact integers from per-pair arithmetic series
    (ATFlash Abstract: the pruned share has a closed form), computed without the
    oracle: a dropped row, an off-by-one distance range or a wrong group threshold
    in the oracle changes these counts."""
    with open(os.path.join(GOLD, "workload_counts.json")) as fh:
        gold = json.load(fh)
    assert len(gold["workloads"]) == 7
    for w in gold["workloads"]:
        got = oracle.count_rows(w["D"], w["base"], w["alpha"], w["g"], w["Nq"], w["Nk"],
                                w["q_pos0"], w["k_pos0"])
        assert got == (w["pruned"], w["total"]), w["name"]


def test_pruned_fraction_grows_logarithmically():
    """Continuum form of the count for a causal N x N square (our derivation of
    the ATFlash Abstract's 'closed form logarithmic in N'):
    fraction ~= (ln(N / (2 pi alpha)) - 3/2) / ln(base) while 2 pi alpha << N <= reach of the
    last pair.  Doubling N adds ~ ln 2 / ln(base)."""
    D, base, alpha = 128, 5e5, 1.0
    prev = None
    for N in (8192, 16384, 32768, 65536, 131072):
        pr, tot = oracle.count_rows(D, base, alpha, 1, N, N)
        frac = pr / tot
        approx = (math.log(N / (2 * math.pi * alpha)) - 1.5) / math.log(base)
        assert abs(frac - approx) < 0.02, (N, frac, approx)
        if prev is not None:
            assert abs((frac - prev) - math.log(2) / math.log(base)) < 0.01
        prev = frac


def test_count_monotone_in_alpha_and_suffix_structure():
    D, base, N = 64, 1e4, 200
    last = None
    for alpha in (0.1, 0.5, 1.0, 2.0, 4.0):
        pr, _ = oracle.count_rows(D, base, alpha, 1, N, N)
        if last is not None:
            assert pr <= last
        last = pr
        T, _ = oracle.thresholds(D, base, alpha, 1)
        assert (np.diff(T) >= 0).all()          # kept set at any d is a suffix of pairs


# ---------------------------------------------------------------------------
# reachability (ATFlash Abstract: every key stays reachable through the
# low-frequency pairs)
# ---------------------------------------------------------------------------

def test_planted_key_is_reachable():
    w = inputs.Workload("plant", "prefill", 1, 4, 2, 128, 2048, 2048, 5e5, 1.0, 1, plant_key=True)
    q, k, v, planted = inputs.prefill_inputs(w, seed=0)
    for (b, hq, t, kvh, j) in planted:
        out, lse = oracle.attention_rows(inputs.bits(q), inputs.bits(k), inputs.bits(v),
                                         Hq=w.Hq, Hkv=w.Hkv, base=w.base, alpha=w.alpha,
                                         g=w.g, scale=w.scale, rows=[(b, hq, t)])
        s = oracle.scores(inputs.bits(q)[b, t, hq], inputs.bits(k)[b, :, kvh], q_pos=t,
                          base=w.base, alpha=w.alpha, g=w.g)
        weight = math.exp(w.scale * s[j] - lse[0])
        assert weight > 0.99, weight
        np.testing.assert_allclose(out[0], v[b, j, kvh].double().numpy(), atol=0.05)


# ---------------------------------------------------------------------------
# decode = the same definition with one query per sequence at kv_len - 1
# ---------------------------------------------------------------------------

def test_decode_rows_match_causal_sdpa_when_window_off():
    B, Hq, Hkv, D, L = 3, 4, 2, 16, 40
    q = _rand((B, Hq, D), 51)
    kc = _rand((B, L, Hkv, D), 52)
    vc = _rand((B, L, Hkv, D), 53)
    kv_len = [40, 1, 17]
    out, lse = oracle.decode_rows(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len,
                                  Hq=Hq, Hkv=Hkv, base=1e4, alpha=float("inf"), g=1, scale=0.25)
    n = 0
    for b in range(B):
        for h in range(Hq):
            kk = kc[b, :kv_len[b], h // (Hq // Hkv)].double()
            vv = vc[b, :kv_len[b], h // (Hq // Hkv)].double()
            z = 0.25 * (kk @ q[b, h].double())
            want = torch.softmax(z, 0) @ vv
            np.testing.assert_allclose(out[n], want.numpy(), atol=1e-10)
            assert abs(lse[n] - float(torch.logsumexp(z, 0))) < 1e-10
            n += 1


# ---------------------------------------------------------------------------
# decode with explicit key positions (ATFlash Abstract: the kept pair set is a
# function of the relative position q_pos - k_pos alone)
# ---------------------------------------------------------------------------

def test_positions_hand_case():
    """D = 4, base 100, alpha 1 (T = (6, 62)), query (1, 2, 3, 4) at position 107.
    Key A = (1, 1, 1, 1) at 100 (d = 7): pair 0 pruned, s = 2 + 4 = 6.
    Key B = (0.5, 0, 0.25, 1) at 0 (d = 107 > 62): both pairs pruned, s = 0.
    Key C = (1, 0, 0, 0) at 107 (d = 0): s = 1.  Key D at 108 is in the future:
    excluded.  Weights (e^6, 1, e, 0) / Z with scale 1."""
    q = _bf16_bits(np.array([1.0, 2.0, 3.0, 4.0]).reshape(1, 1, 4))
    kk = np.zeros((1, 4, 1, 4))
    vv = np.zeros((1, 4, 1, 4))
    kk[0, 0, 0] = [1.0, 1.0, 1.0, 1.0]
    kk[0, 1, 0] = [0.5, 0.0, 0.25, 1.0]
    kk[0, 2, 0] = [1.0, 0.0, 0.0, 0.0]
    kk[0, 3, 0] = [9.0, 9.0, 9.0, 9.0]
    vv[0, 0, 0] = [1.0, 0.0, 0.0, 0.0]
    vv[0, 1, 0] = [0.0, 1.0, 0.0, 0.0]
    vv[0, 2, 0] = [0.0, 0.0, 1.0, 0.0]
    vv[0, 3, 0] = [0.0, 0.0, 0.0, 1.0]
    out, lse = oracle.decode_positions(q, _bf16_bits(kk), _bf16_bits(vv), [4], [107],
                                       [[100, 0, 107, 108]], Hq=1, Hkv=1, base=100.0,
                                       alpha=1.0, g=1, scale=1.0)
    z = math.exp(6.0) + 1.0 + math.exp(1.0)
    np.testing.assert_allclose(out[0], [math.exp(6.0) / z, 1.0 / z, math.e / z, 0.0],
                               rtol=0, atol=1e-12)
    assert abs(lse[0] - math.log(z)) < 1e-12


def test_positions_alpha_inf_is_masked_sdpa():
    """alpha = inf: ordinary attention under the mask k_pos <= q_pos."""
    B, Hq, Hkv, D, L = 2, 4, 2, 16, 30
    q = _rand((B, Hq, D), 61)
    kc = _rand((B, L, Hkv, D), 62)
    vc = _rand((B, L, Hkv, D), 63)
    rng = np.random.default_rng(5)
    kv_len = [30, 19]
    k_pos = rng.integers(0, 500, size=(B, L))
    q_pos = [400, 250]
    out, lse = oracle.decode_positions(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len,
                                       q_pos, k_pos, Hq=Hq, Hkv=Hkv, base=1e4,
                                       alpha=float("inf"), g=1, scale=0.25)
    n = 0
    for b in range(B):
        keep = torch.tensor(k_pos[b, :kv_len[b]] <= q_pos[b])
        for h in range(Hq):
            kk = kc[b, :kv_len[b], h // (Hq // Hkv)].double()
            vv = vc[b, :kv_len[b], h // (Hq // Hkv)].double()
            z = 0.25 * (kk @ q[b, h].double())
            z = torch.where(keep, z, torch.tensor(-math.inf, dtype=torch.float64))
            want = torch.softmax(z, 0) @ vv
            np.testing.assert_allclose(out[n], want.numpy(), atol=1e-10)
            assert abs(lse[n] - float(torch.logsumexp(z, 0))) < 1e-10
            n += 1


def test_positions_contiguous_equal_decode_rows():
    """k_pos = 0..n-1 with the query at n-1 is plain decode."""
    B, Hq, Hkv, D, L = 3, 4, 1, 32, 300
    q = _rand((B, Hq, D), 71)
    kc = _rand((B, L, Hkv, D), 72)
    vc = _rand((B, L, Hkv, D), 73)
    kv_len = [300, 1, 137]
    k_pos = np.tile(np.arange(L), (B, 1))
    a = oracle.decode_positions(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len,
                                [n - 1 for n in kv_len], k_pos, Hq=Hq, Hkv=Hkv, base=1e4,
                                alpha=1.0, g=1, scale=0.2)
    b = oracle.decode_rows(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len, Hq=Hq,
                           Hkv=Hkv, base=1e4, alpha=1.0, g=1, scale=0.2)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("g", [1, 8])
def test_positions_joint_permutation_invariance(g):
    """Reordering the cache rows together with their positions changes nothing
    but the summation order; a position-only shift of everything by the same
    offset changes nothing at all (relative positions are unchanged)."""
    B, Hq, Hkv, D, L = 1, 2, 1, 32, 400
    q = _rand((B, Hq, D), 81)
    kc = _rand((B, L, Hkv, D), 82)
    vc = _rand((B, L, Hkv, D), 83)
    rng = np.random.default_rng(9)
    k_pos = np.sort(rng.choice(5000, size=L, replace=False))[None, :]
    q_pos = [int(k_pos[0, -1]) + 3]
    kw = dict(Hq=Hq, Hkv=Hkv, base=1e4, alpha=1.0, g=g, scale=0.3)
    o1, l1 = oracle.decode_positions(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), [L],
                                     q_pos, k_pos, **kw)
    perm = rng.permutation(L)
    o2, l2 = oracle.decode_positions(inputs.bits(q), inputs.bits(kc)[:, perm],
                                     inputs.bits(vc)[:, perm], [L], q_pos, k_pos[:, perm], **kw)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-12)
    o3, l3 = oracle.decode_positions(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), [L],
                                     [q_pos[0] + 12345], k_pos + 12345, **kw)
    np.testing.assert_array_equal(o3, o1)
    np.testing.assert_array_equal(l3, l1)
    # and the windowed result differs from the window-off one (the pin is not vacuous)
    o4, _ = oracle.decode_positions(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), [L],
                                    q_pos, k_pos, **dict(kw, alpha=float("inf")))
    assert np.abs(o4 - o1).max() > 1e-3


# ---------------------------------------------------------------------------
# block mask stacked on the window (ATFlash Abstract: the window composes with
# token-level selection)
# ---------------------------------------------------------------------------

def test_block_mask_hand_case():
    """The 2-pair case of test_two_pair_softmax_by_hand (query at 7, T = (6, 62)) with
    4-key blocks.  Mask (0, 1): keys 4..7 remain, scores (0, 0, 0, 5.25).  Mask (1, 0):
    keys 0..3 remain, scores (6, 0, 0, 0) (the row's own key is masked out)."""
    q = _bf16_bits(np.array([1.0, 2.0, 3.0, 4.0]).reshape(1, 1, 1, 4))
    kk = np.zeros((1, 8, 1, 4))
    vv = np.zeros((1, 8, 1, 4))
    kk[0, 0, 0] = [1.0, 1.0, 1.0, 1.0]
    kk[0, 7, 0] = [0.5, 0.0, 0.25, 1.0]
    vv[0, 0, 0] = [1.0, 0.0, 0.0, 0.0]
    vv[0, 7, 0] = [0.0, 1.0, 0.0, 0.0]
    vv[0, 1:7, 0, 2] = 1.0
    kw = dict(Hq=1, Hkv=1, q_pos0=7, k_pos0=0, base=100.0, alpha=1.0, g=1, scale=1.0,
              rows=[(0, 0, 0)], block_q=1, block_k=4)
    out, lse = oracle.attention_rows_masked(q, _bf16_bits(kk), _bf16_bits(vv),
                                            np.array([0, 1]).reshape(1, 1, 1, 2), **kw)
    z = 3.0 + math.exp(5.25)
    np.testing.assert_allclose(out[0], [0.0, math.exp(5.25) / z, 3.0 / z, 0.0], rtol=0, atol=1e-12)
    assert abs(lse[0] - math.log(z)) < 1e-12
    out, lse = oracle.attention_rows_masked(q, _bf16_bits(kk), _bf16_bits(vv),
                                            np.array([1, 0]).reshape(1, 1, 1, 2), **kw)
    z = math.exp(6.0) + 3.0
    np.testing.assert_allclose(out[0], [math.exp(6.0) / z, 0.0, 3.0 / z, 0.0], rtol=0, atol=1e-12)
    assert abs(lse[0] - math.log(z)) < 1e-12
    out, lse = oracle.attention_rows_masked(q, _bf16_bits(kk), _bf16_bits(vv),
                                            np.zeros((1, 1, 1, 2)), **kw)
    assert (out == 0).all() and lse[0] == -math.inf


def test_block_mask_all_ones_is_attention_rows():
    q = _rand((2, 70, 2, 16), 91)
    k = _rand((2, 70, 1, 16), 92)
    v = _rand((2, 70, 1, 16), 93)
    rows = [(b, h, t) for b in range(2) for h in range(2) for t in range(0, 70, 3)]
    kw = dict(Hq=2, Hkv=1, base=1e4, alpha=1.0, g=1, scale=0.25, rows=rows)
    a = oracle.attention_rows(inputs.bits(q), inputs.bits(k), inputs.bits(v), **kw)
    m = np.ones((2, 2, 3, 5), dtype=np.uint8)
    b = oracle.attention_rows_masked(inputs.bits(q), inputs.bits(k), inputs.bits(v), m,
                                     block_q=32, block_k=16, **kw)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_block_mask_alpha_inf_is_masked_sdpa():
    """alpha = inf: ordinary attention under (causal AND block mask), by a library routine."""
    B, Nq, Nk, Hq, Hkv, D, q0, k0 = 2, 40, 56, 2, 1, 16, 16, 0
    q = _rand((B, Nq, Hq, D), 94)
    k = _rand((B, Nk, Hkv, D), 95)
    v = _rand((B, Nk, Hkv, D), 96)
    bq, bk = 8, 8
    rng = np.random.default_rng(3)
    m = (rng.random((B, Hq, Nq // bq, Nk // bk)) < 0.5).astype(np.uint8)
    rows = [(b, h, t) for b in range(B) for h in range(Hq) for t in range(Nq)]
    out, lse = oracle.attention_rows_masked(inputs.bits(q), inputs.bits(k), inputs.bits(v), m,
                                            Hq=Hq, Hkv=Hkv, q_pos0=q0, k_pos0=k0, base=1e4,
                                            alpha=float("inf"), g=1, scale=0.25, rows=rows,
                                            block_q=bq, block_k=bk)
    qf = q.double().permute(0, 2, 1, 3)
    kf = k.double().repeat_interleave(Hq // Hkv, dim=2).permute(0, 2, 1, 3)
    vf = v.double().repeat_interleave(Hq // Hkv, dim=2).permute(0, 2, 1, 3)
    causal = (k0 + torch.arange(Nk))[None, :] <= (q0 + torch.arange(Nq))[:, None]
    blk = torch.tensor(m, dtype=torch.bool).repeat_interleave(bq, 2).repeat_interleave(bk, 3)
    allowed = causal[None, None] & blk
    z = 0.25 * qf @ kf.transpose(-1, -2)
    z = torch.where(allowed, z, torch.tensor(-math.inf, dtype=torch.float64))
    for n, (b, h, t) in enumerate(rows):
        if not allowed[b, h, t].any():
            assert lse[n] == -math.inf and (out[n] == 0).all()
            continue
        want = torch.softmax(z[b, h, t], 0) @ vf[b, h]
        np.testing.assert_allclose(out[n], want.numpy(), atol=1e-10)
        assert abs(lse[n] - float(torch.logsumexp(z[b, h, t], 0))) < 1e-10
    assert (~allowed.reshape(-1, Nk).any(1)).any()     # some rows are empty: the case is covered


# ---------------------------------------------------------------------------
# RoPE (WavePrune, Original abstract: 2-D channels rotated at channel-specific
# frequencies; logits depend on the position difference only)
# ---------------------------------------------------------------------------

def _bf16_values(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def test_rope_hand_cases():
    # D = 2: one pair, theta_0 = 1 whatever the base
    x = _bf16_bits(np.array([[[1.0, 0.0]], [[0.0, 1.0]]]))
    y = oracle.rope(x, [1, 2], base=1e4, exact=True)
    np.testing.assert_allclose(y[0, 0], [math.cos(1.0), math.sin(1.0)], rtol=0, atol=1e-15)
    np.testing.assert_allclose(y[1, 0], [-math.sin(2.0), math.cos(2.0)], rtol=0, atol=1e-15)
    # D = 4, base 100: theta = (1, 0.1); position 10 turns pair 0 by 10 rad and pair 1 by 1 rad
    x = _bf16_bits(np.array([[[1.0, 2.0, 0.0, 0.0]]]))
    y = oracle.rope(x, [10], base=100.0, exact=True)
    np.testing.assert_allclose(y[0, 0], [math.cos(10.0), 2 * math.cos(1.0), math.sin(10.0),
                                         2 * math.sin(1.0)], rtol=0, atol=1e-14)


def test_rope_position_zero_is_identity_and_pairs_are_half_split():
    x = _rand((5, 3, 64), 201)
    xb = inputs.bits(x)
    assert np.array_equal(oracle.rope(xb, [0] * 5, base=1e4), xb)
    e = np.zeros((1, 1, 16)); e[0, 0, 0] = 1.0
    y = oracle.rope(_bf16_bits(e), [3], base=1e4, exact=True)[0, 0]
    assert (y[[i for i in range(16) if i not in (0, 8)]] == 0).all()
    assert y[0] != 0 and y[8] != 0


def test_rope_preserves_pair_norms_and_depends_on_relative_position():
    D, n = 64, 6
    q = inputs.bits(_rand((n, 1, D), 202))
    k = inputs.bits(_rand((n, 1, D), 203))
    P = D // 2
    rng = np.random.default_rng(4)
    m = rng.integers(0, 100000, n)
    nn = rng.integers(0, 100000, n)
    shift = 123457
    yq = oracle.rope(q, m, base=5e5, exact=True)
    yk = oracle.rope(k, nn, base=5e5, exact=True)
    yq2 = oracle.rope(q, m + shift, base=5e5, exact=True)
    yk2 = oracle.rope(k, nn + shift, base=5e5, exact=True)
    xq = _bf16_values(q)
    np.testing.assert_allclose(yq[..., :P] ** 2 + yq[..., P:] ** 2,
                               xq[..., :P] ** 2 + xq[..., P:] ** 2, rtol=1e-12)
    # per pair: the rotated product depends on m - n only
    s1 = yq[..., :P] * yk[..., :P] + yq[..., P:] * yk[..., P:]
    s2 = yq2[..., :P] * yk2[..., :P] + yq2[..., P:] * yk2[..., P:]
    np.testing.assert_allclose(s1, s2, rtol=0, atol=1e-9)


def test_rope_rounds_to_nearest_bf16():
    """Each bf16 output is the representable value nearest the exact result."""
    x = inputs.bits(_rand((64, 4, 128), 204))
    pos = np.arange(64) * 977
    yb = oracle.rope(x, pos, base=1e6).astype(np.uint32)
    ye = oracle.rope(x, pos, base=1e6, exact=True)
    b = _bf16_values(yb)
    up = _bf16_values((yb + 1) & 0xFFFF)       # next magnitude up (same sign)
    dn = _bf16_values(np.where((yb & 0x7FFF) == 0, yb, yb - 1))
    err = np.abs(ye - b)
    assert (err <= np.abs(ye - up)).all() and (err <= np.abs(ye - dn)).all()
    assert (np.sign(b) == np.sign(ye))[ye != 0].all()


# ---------------------------------------------------------------------------
# prefill with explicit per-token positions (ATFlash Abstract: the window is a
# function of the relative position)
# ---------------------------------------------------------------------------

def test_prefill_positions_contiguous_equal_attention_rows():
    B, Nq, Nk, Hq, Hkv, D, q0, k0 = 2, 30, 50, 2, 1, 16, 40, 17
    q = _rand((B, Nq, Hq, D), 301)
    k = _rand((B, Nk, Hkv, D), 302)
    v = _rand((B, Nk, Hkv, D), 303)
    rows = [(b, h, t) for b in range(B) for h in range(Hq) for t in range(Nq)]
    kw = dict(Hq=Hq, Hkv=Hkv, base=100.0, alpha=1.0, g=1, scale=0.3, rows=rows)
    a = oracle.attention_rows(inputs.bits(q), inputs.bits(k), inputs.bits(v), q_pos0=q0, k_pos0=k0, **kw)
    qp = np.tile(q0 + np.arange(Nq), (B, 1))
    kp = np.tile(k0 + np.arange(Nk), (B, 1))
    b = oracle.attention_positions(inputs.bits(q), inputs.bits(k), inputs.bits(v), qp, kp, **kw)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_prefill_positions_hand_case():
    """Query (1, 2, 3, 4) at position 50 (D = 4, base 100, T = (6, 62)); keys at 0, 45, 50 and 51:
    d = 50 (pair 0 pruned: s = 2 + 4 = 6 for k = (1, 1, 1, 1)), d = 5 (both kept: s = 1 for
    k = (1, 0, 0, 0)), d = 0 (s = 0 for k = 0), d = -1 (future: left out)."""
    q = _bf16_bits(np.array([1.0, 2.0, 3.0, 4.0]).reshape(1, 1, 1, 4))
    kk = np.zeros((1, 4, 1, 4))
    vv = np.eye(4).reshape(1, 4, 1, 4)
    kk[0, 0, 0] = [1.0, 1.0, 1.0, 1.0]
    kk[0, 1, 0] = [1.0, 0.0, 0.0, 0.0]
    kk[0, 3, 0] = [9.0, 9.0, 9.0, 9.0]
    out, lse = oracle.attention_positions(q, _bf16_bits(kk), _bf16_bits(vv), [[50]],
                                          [[0, 45, 50, 51]], Hq=1, Hkv=1, base=100.0, alpha=1.0,
                                          g=1, scale=1.0, rows=[(0, 0, 0)])
    z = math.exp(6.0) + math.e + 1.0
    np.testing.assert_allclose(out[0], [math.exp(6.0) / z, math.e / z, 1.0 / z, 0.0], rtol=0,
                               atol=1e-12)
    assert abs(lse[0] - math.log(z)) < 1e-12


def test_prefill_positions_alpha_inf_is_masked_sdpa_and_shift_invariant():
    B, Nq, Nk, Hq, Hkv, D = 2, 24, 40, 2, 2, 16
    q = _rand((B, Nq, Hq, D), 304)
    k = _rand((B, Nk, Hkv, D), 305)
    v = _rand((B, Nk, Hkv, D), 306)
    rng = np.random.default_rng(8)
    kp = np.sort(rng.integers(0, 300, (B, Nk)), axis=1)
    qp = np.sort(rng.integers(0, 300, (B, Nq)), axis=1)
    rows = [(b, h, t) for b in range(B) for h in range(Hq) for t in range(Nq)]
    out, lse = oracle.attention_positions(inputs.bits(q), inputs.bits(k), inputs.bits(v), qp, kp,
                                          Hq=Hq, Hkv=Hkv, base=1e4, alpha=float("inf"), g=1,
                                          scale=0.25, rows=rows)
    for n, (b, h, t) in enumerate(rows):
        allowed = torch.tensor(kp[b] <= qp[b, t])
        if not allowed.any():
            assert lse[n] == -math.inf and (out[n] == 0).all()
            continue
        z = 0.25 * (k[b, :, h].double() @ q[b, t, h].double())
        z = torch.where(allowed, z, torch.tensor(-math.inf, dtype=torch.float64))
        np.testing.assert_allclose(out[n], (torch.softmax(z, 0) @ v[b, :, h].double()).numpy(),
                                   atol=1e-10)
    kw = dict(Hq=Hq, Hkv=Hkv, base=1e4, alpha=1.0, g=8, scale=0.25, rows=rows)
    a = oracle.attention_positions(inputs.bits(q), inputs.bits(k), inputs.bits(v), qp, kp, **kw)
    b2 = oracle.attention_positions(inputs.bits(q), inputs.bits(k), inputs.bits(v), qp + 99991,
                                    kp + 99991, **kw)
    np.testing.assert_array_equal(a[0], b2[0])
