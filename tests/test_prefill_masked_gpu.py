"""Prefill under a 128 x 128 block mask stacked on the window, through the C ABI:
the mask packing (bit-exact), an all-ones mask (bitwise equal to the unmasked
call), random and structured masks against the oracle, masks that leave query
tiles or whole CTAs without a key, and CTAs with no causal key at all."""
import math

import numpy as np
import pytest
import torch

import oracle
import rope_wavelength_sparsity_b200 as wp
from rope_wavelength_sparsity_b200 import inputs

from _parity import check_rows

pytestmark = pytest.mark.gpu

BLK = wp.MASK_BLOCK


def _qkv(B, Nq, Nk, Hq, Hkv, D, seed):
    return (inputs.randn_bf16((B, Nq, Hq, D), 100 * seed + 1),
            inputs.randn_bf16((B, Nk, Hkv, D), 100 * seed + 2),
            inputs.randn_bf16((B, Nk, Hkv, D), 100 * seed + 3))


def _nblocks(Nq, Nk):
    return -(-Nq // BLK), -(-Nk // BLK)


def _random_mask(B, Hq, Nq, Nk, density, seed, keep_diagonal=True, q_pos0=0, k_pos0=0):
    nqb, nkb = _nblocks(Nq, Nk)
    g = torch.Generator().manual_seed(seed)
    m = torch.rand((B, Hq, nqb, nkb), generator=g) < density
    if keep_diagonal:
        for qb in range(nqb):
            kb = min((q_pos0 - k_pos0 + qb * BLK) // BLK, nkb - 1)
            if kb >= 0:
                m[:, :, qb, kb] = True
    return m


def _check_all_rows(q, k, v, m, *, D, g, alpha, base, Hq, Hkv, q_pos0=0, k_pos0=0, rows=None,
                    what=""):
    B, Nq = q.shape[0], q.shape[1]
    win = wp.Window(D, base, alpha, g)
    out, lse = wp.prefill_masked(q.cuda(), k.cuda(), v.cuda(), m.cuda(), win, q_pos0=q_pos0,
                                 k_pos0=k_pos0)
    assert wp.device_status() == wp.OK
    if rows is None:
        rows = [(b, h, t) for b in range(B) for h in range(Hq) for t in range(Nq)]
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    o_ref, l_ref = oracle.attention_rows_masked(inputs.bits(q), inputs.bits(k), inputs.bits(v),
                                                m.numpy(), Hq=Hq, Hkv=Hkv, q_pos0=q_pos0,
                                                k_pos0=k_pos0, base=base, alpha=alpha, g=g,
                                                scale=1.0 / math.sqrt(D), rows=rows,
                                                block_q=BLK, block_k=BLK)
    bi, hi, ti = (torch.as_tensor(rows[:, i]) for i in range(3))
    return check_rows(out.float().cpu()[bi, ti, hi].numpy(), lse.cpu()[bi, hi, ti].numpy(),
                      o_ref, l_ref, what)


@pytest.mark.parametrize("shape", [(1, 1, 1, 1), (2, 3, 4, 33), (1, 2, 128, 300), (3, 1, 5, 64)])
def test_pack_block_mask_bit_exact(cuda_dev, shape):
    g = torch.Generator().manual_seed(sum(shape))
    m = torch.rand(shape, generator=g) < 0.4
    words = wp.pack_block_mask(m.cuda())
    torch.cuda.synchronize()
    bits = m.numpy().astype(np.uint64)
    nw = -(-shape[3] // 32)
    want = np.zeros(shape[:3] + (nw,), dtype=np.uint64)
    for kb in range(shape[3]):
        want[..., kb // 32] |= bits[..., kb] << np.uint64(kb % 32)
    assert np.array_equal(words.cpu().numpy().view(np.uint32).astype(np.uint64), want)


@pytest.mark.parametrize("D,g", [(64, 8), (128, 1)])
def test_all_ones_mask_equals_unmasked(cuda_dev, D, g):
    B, Nq, Nk, Hq, Hkv = 1, 700, 900, 4, 2
    q, k, v = _qkv(B, Nq, Nk, Hq, Hkv, D, seed=3)
    win = wp.Window(D, 1e4, 1.0, g)
    nqb, nkb = _nblocks(Nq, Nk)
    m = torch.ones((B, Hq, nqb, nkb), dtype=torch.bool)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    a = wp.prefill_masked(qd, kd, vd, m.cuda(), win, q_pos0=200)
    b = wp.prefill(qd, kd, vd, win, q_pos0=200)
    assert wp.device_status() == wp.OK
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


CASES = [
    # D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q_pos0, k_pos0, density
    (128, 1, 1.0, 5e5, 1, 3, 1, 700, 700, 0, 0, 0.5),
    (64, 8, 1.0, 1e6, 2, 4, 2, 520, 520, 0, 0, 0.4),
    (128, 8, 1.0, 1e7, 1, 2, 2, 300, 1500, 1200, 0, 0.3),     # chunked prefill
    (64, 1, 2.0, 1e4, 1, 2, 1, 1000, 1000, 0, 0, 0.7),
    (128, 1, 0.3, 1e4, 1, 2, 1, 650, 650, 0, 0, 0.5),         # many corrected tiles
    (64, 1, 1.0, 10.0, 1, 2, 2, 333, 333, 0, 0, 0.6),
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_random_block_masks_vs_oracle(cuda_dev, case):
    D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q0, k0, density = case
    q, k, v = _qkv(B, Nq, Nk, Hq, Hkv, D, seed=len(str(case)))
    m = _random_mask(B, Hq, Nq, Nk, density, seed=len(str(case)), q_pos0=q0, k_pos0=k0)
    _check_all_rows(q, k, v, m, D=D, g=g, alpha=alpha, base=base, Hq=Hq, Hkv=Hkv, q_pos0=q0,
                    k_pos0=k0, what=str(case))


def test_masks_without_diagonal_and_empty_tiles(cuda_dev):
    """Query tiles whose every attended tile lies in the future or is masked out,
    a CTA (two query tiles) with nothing attended, and a head with an all-zero mask."""
    D, B, Hq, Hkv, Nq, Nk = 64, 1, 3, 1, 900, 900
    q, k, v = _qkv(B, Nq, Nk, Hq, Hkv, D, seed=9)
    nqb, nkb = _nblocks(Nq, Nk)
    m = _random_mask(B, Hq, Nq, Nk, 0.5, seed=4, keep_diagonal=False)
    m[0, 0, 2:4, :] = False          # the second CTA of head 0 attends nothing
    m[0, 1, 5, 6:] = True            # only future tiles for query tile 5
    m[0, 1, 5, :6] = False
    m[0, 2] = False                  # head 2: nothing at all
    _check_all_rows(q, k, v, m, D=D, g=1, alpha=1.0, base=1e4, Hq=Hq, Hkv=Hkv,
                    what="empty tiles")


def test_vertical_slash_pattern_sampled(cuda_dev):
    """A MInference-style pattern at 8K: a few 'vertical' key tiles every query
    tile attends plus a band of 'slash' tiles along the diagonal; sampled rows."""
    D, g, B, Hq, Hkv, N = 128, 1, 1, 4, 1, 8192
    q, k, v = _qkv(B, N, N, Hq, Hkv, D, seed=12)
    nqb, nkb = _nblocks(N, N)
    m = torch.zeros((B, Hq, nqb, nkb), dtype=torch.bool)
    for h in range(Hq):
        m[0, h, :, [0, 1, 17 + h, 40]] = True
        for qb in range(nqb):
            m[0, h, qb, max(0, qb - 3 - h):qb + 1] = True
    rng = np.random.default_rng(2)
    rows = [(0, int(rng.integers(0, Hq)), int(t)) for t in
            np.concatenate([[0, 127, 128, 4095, 4096, N - 1], rng.integers(0, N, 58)])]
    _check_all_rows(q, k, v, m, D=D, g=g, alpha=1.0, base=5e5, Hq=Hq, Hkv=Hkv, rows=rows,
                    what="vertical-slash")


def test_prefill_without_any_causal_key(cuda_dev):
    """Nk = 0, and keys that all sit after a whole CTA's queries: empty rows and no
    timeout (the CTA loads nothing and waits for nothing)."""
    D, Hq = 64, 2
    win = wp.Window(D, 1e4, 1.0, 1)
    q = inputs.randn_bf16((1, 300, Hq, D), 1).cuda()
    k = inputs.randn_bf16((1, 0, 1, D), 2).cuda()
    out, lse = wp.prefill(q, k, k, win)
    assert wp.device_status() == wp.OK
    assert (out.float() == 0).all() and torch.isneginf(lse).all()
    k = inputs.randn_bf16((1, 200, 1, D), 3)
    v = inputs.randn_bf16((1, 200, 1, D), 4)
    qc = inputs.randn_bf16((1, 600, Hq, D), 5)
    # keys at 400..599: the first CTA's rows 0..255 see none of them
    out, lse = wp.prefill(qc.cuda(), k.cuda(), v.cuda(), win, q_pos0=0, k_pos0=400)
    assert wp.device_status() == wp.OK
    assert (out[0, :256].float() == 0).all() and torch.isneginf(lse[0, :, :256]).all()
    rows = [(0, h, t) for h in range(Hq) for t in (399, 400, 401, 599)]
    o_ref, l_ref = oracle.attention_rows(inputs.bits(qc), inputs.bits(k), inputs.bits(v), Hq=Hq,
                                         Hkv=1, q_pos0=0, k_pos0=400, base=1e4, alpha=1.0, g=1,
                                         scale=1.0 / math.sqrt(D), rows=rows)
    check_rows(np.stack([out[0, t, h].float().cpu().numpy() for (_, h, t) in rows]),
               np.array([float(lse[0, h, t]) for (_, h, t) in rows]), o_ref, l_ref, "late keys")


def test_prefill_masked_rejects_short_rows(cuda_dev):
    D = 64
    q = inputs.randn_bf16((1, 100, 1, D), 1).cuda()
    k = inputs.randn_bf16((1, 5000, 1, D), 2).cuda()   # 40 key tiles: 2 words per row
    words = torch.zeros((1, 1, 1, 1), dtype=torch.int32, device="cuda")
    with pytest.raises(wp.WpattnError) as e:
        wp.prefill_masked(q, k, k, words, wp.Window(D, 1e4, 1.0, 1), q_pos0=4900)
    assert e.value.code == wp.EINVAL
