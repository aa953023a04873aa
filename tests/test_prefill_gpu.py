"""Prefill parity on the GPU: CUDA path (through the C ABI) vs the oracle,
every output row, at sizes that span several 128-row tiles and a ragged
tail, plus the edge cases of the method (window off, every pair pruned,
partial k-steps, chunked prefill, rows without any causal key)."""
import math

import pytest
import torch

import rope_wavelength_sparsity_b200 as wp
from rope_wavelength_sparsity_b200 import inputs

from _parity import prefill_parity

pytestmark = pytest.mark.gpu


def _qkv(B, Nq, Nk, Hq, Hkv, D, seed):
    q = inputs.randn_bf16((B, Nq, Hq, D), 100 * seed + 1)
    k = inputs.randn_bf16((B, Nk, Hkv, D), 100 * seed + 2)
    v = inputs.randn_bf16((B, Nk, Hkv, D), 100 * seed + 3)
    return q, k, v


def test_tiny_workload_all_rows(cuda_dev):
    w = inputs.WORKLOADS["tiny"]
    for seed in range(4):
        q, k, v, _ = inputs.prefill_inputs(w, seed=seed)
        prefill_parity(q, k, v, Hq=w.Hq, Hkv=w.Hkv, D=w.D, base=w.base, alpha=w.alpha, g=w.g,
                       what=f"tiny seed {seed}")


CASES = [
    # D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q_pos0, k_pos0
    (128, 1, 1.0, 5e5, 1, 3, 1, 300, 300, 0, 0),        # GQA 3, ragged tail
    (64, 8, 1.0, 1e6, 2, 7, 1, 257, 257, 0, 0),         # GQA 7, g = 8, batch 2
    (128, 8, 1.0, 1e7, 1, 2, 2, 100, 700, 600, 0),      # chunked prefill, Nq < 128
    (64, 1, float("inf"), 1e4, 1, 2, 1, 384, 384, 0, 0),  # window off
    (128, 1, 2.0, 5e5, 1, 2, 2, 520, 520, 0, 0),        # alpha = 2
    (64, 1, 1e-3, 1e4, 1, 1, 1, 400, 400, 0, 0),        # far tiles: every pair pruned
    (64, 1, 1.0, 10.0, 1, 2, 1, 333, 333, 0, 0),        # many thresholds inside a tile
    (128, 1, 0.3, 1e4, 1, 2, 1, 450, 450, 0, 0),        # partial k-steps everywhere
    (128, 1, 1.0, 5e5, 1, 1, 1, 50, 50, 0, 0),          # one tile, Nk < 128
    (64, 1, 1.0, 1e4, 1, 2, 2, 200, 150, 0, 60),        # first 60 rows see no key
    (128, 8, 2.0, 1e4, 1, 16, 1, 130, 1000, 870, 0),    # GQA 16, q_pos0 off the tile grid
    (64, 8, 0.05, 1e4, 1, 2, 1, 600, 600, 0, 0),        # g = 8 group boundaries inside tiles
    (128, 1, 1.0, 5e5, 1, 1, 1, 1, 1, 0, 0),            # one query, one key
    (64, 1, 1.0, 1e4, 1, 1, 1, 129, 129, 0, 0),         # one row into a second tile
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_prefill_cases_all_rows(cuda_dev, case):
    D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q0, k0 = case
    q, k, v = _qkv(B, Nq, Nk, Hq, Hkv, D, seed=len(str(case)))
    prefill_parity(q, k, v, Hq=Hq, Hkv=Hkv, D=D, base=base, alpha=alpha, g=g, q_pos0=q0,
                   k_pos0=k0, what=str(case))


# More edges of the D = 64, g = 8 shape: large logits (the running max jumps,
# so O is rescaled), a chunk at the end of the keys, the window off, a CTA whose
# second query tile is empty, rows that see no key, group edges inside tiles.
G8_EDGE_CASES = [
    # D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q0, k0, input scale
    (64, 8, 1.0, 1e6, 1, 2, 1, 1000, 1000, 0, 0, 3.0),     # large logits: the lazy O rescale
    (64, 8, 1.0, 1e6, 1, 3, 1, 300, 1500, 1200, 0, 3.0),   # chunk at the end of the keys
    (64, 8, float("inf"), 1e6, 1, 2, 2, 700, 700, 0, 0, 1.0),  # window off
    (64, 8, 1.0, 1e4, 1, 2, 1, 100, 900, 800, 0, 1.0),     # second query tile empty
    (64, 8, 1.0, 1e4, 1, 2, 1, 200, 200, 0, 60, 2.0),      # first rows see no key
    (64, 8, 0.05, 1e4, 2, 4, 2, 513, 513, 0, 0, 3.0),      # group edges inside tiles, batch 2
]


@pytest.mark.parametrize("case", G8_EDGE_CASES, ids=[str(i) for i in range(len(G8_EDGE_CASES))])
def test_prefill_g8_edges_all_rows(cuda_dev, case):
    D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q0, k0, amp = case
    q, k, v = _qkv(B, Nq, Nk, Hq, Hkv, D, seed=len(str(case)) + 500)
    # q and k scaled up: large logits, so the running max jumps and O is rescaled;
    # v scaled down by the same factor: with near one-hot rows the bf16 rounding of
    # P (relative 2^-8) times max |v| must stay inside the output tolerance
    q = (q.float() * amp).to(torch.bfloat16)
    k = (k.float() * amp).to(torch.bfloat16)
    v = (v.float() / amp).to(torch.bfloat16)
    prefill_parity(q, k, v, Hq=Hq, Hkv=Hkv, D=D, base=base, alpha=alpha, g=g, q_pos0=q0,
                   k_pos0=k0, what=str(case))


def test_planted_key_small(cuda_dev):
    w = inputs.Workload("plant", "prefill", 1, 8, 2, 128, 1500, 1500, 5e5, 1.0, 1, plant_key=True)
    q, k, v, planted = inputs.prefill_inputs(w, seed=3)
    rows = [(b, hq, t) for (b, hq, t, _, _) in planted] + [(0, h, t) for h in range(8)
                                                            for t in (0, 700, 1499)]
    prefill_parity(q, k, v, Hq=w.Hq, Hkv=w.Hkv, D=w.D, base=w.base, alpha=w.alpha, g=w.g,
                   rows=rows, what="planted")
    out, _ = wp.prefill(q.cuda(), k.cuda(), v.cuda(), wp.Window(w.D, w.base, w.alpha, w.g))
    for (b, hq, t, kvh, j) in planted:
        assert torch.allclose(out[b, t, hq].float().cpu(), v[b, j, kvh].float(), atol=0.05)


def test_prefill_deterministic(cuda_dev):
    q, k, v = _qkv(1, 700, 700, 4, 2, 128, seed=9)
    win = wp.Window(128, 5e5, 1.0, 1)
    o1, l1 = wp.prefill(q.cuda(), k.cuda(), v.cuda(), win)
    o2, l2 = wp.prefill(q.cuda(), k.cuda(), v.cuda(), win)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_prefill_without_lse_and_custom_scale(cuda_dev):
    q, k, v = _qkv(1, 200, 200, 2, 1, 64, seed=4)
    win = wp.Window(64, 1e4, 1.0, 1)
    o1, _ = wp.prefill(q.cuda(), k.cuda(), v.cuda(), win, want_lse=False, scale=0.2)
    o2, _ = wp.prefill(q.cuda(), k.cuda(), v.cuda(), win, scale=0.2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    prefill_parity(q, k, v, Hq=2, Hkv=1, D=64, base=1e4, alpha=1.0, g=1, scale=0.2, what="scale")


def test_prefill_rejects_non_sm100_or_bad_args_gracefully(cuda_dev):
    q, k, v = _qkv(1, 8, 8, 2, 1, 64, seed=5)
    with pytest.raises(wp.WpattnError):
        wp.prefill(q.cuda(), k.cuda(), v.cuda(), wp.Window(64, 1e4, -1.0, 1))
