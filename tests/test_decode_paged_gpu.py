"""Decode with explicit key positions and from a paged cache, through the C ABI.

Positions: against the oracle's decode with positions (evicted, shuffled and
partly-future key positions), and bitwise against plain decode when the
positions are the contiguous ones.  Paged: bitwise against decode on the
cache the block table describes (same arithmetic in the same order), and
against the oracle; unused pool rows are NaN, so a read of one shows.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import rope_wavelength_sparsity_b200 as wp
from rope_wavelength_sparsity_b200 import inputs

from _parity import check_rows
from test_decode_gpu import CASES

pytestmark = pytest.mark.gpu


def _oracle_positions(q, kc, vc, kv_len, q_pos, k_pos, *, Hq, Hkv, D, base, alpha, g, scale):
    return oracle.decode_positions(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len,
                                   q_pos, k_pos.numpy().astype(np.int64), Hq=Hq, Hkv=Hkv,
                                   base=base, alpha=alpha, g=g, scale=scale)


def _all_rows(out, lse, B, Hq):
    oc, lc = out.float().cpu(), lse.cpu()
    rows = [(b, h) for b in range(B) for h in range(Hq)]
    return (np.stack([oc[b, h].numpy() for (b, h) in rows]),
            np.array([float(lc[b, h]) for (b, h) in rows]))


@pytest.mark.parametrize("case", CASES[:6], ids=[str(i) for i in range(6)])
def test_contiguous_positions_equal_decode(cuda_dev, case):
    D, g, alpha, base, B, Hq, Hkv, L, kv_len = case
    seed = len(str(case)) + 700
    q = inputs.randn_bf16((B, Hq, D), seed * 10 + 1).cuda()
    kc = inputs.randn_bf16((B, L, Hkv, D), seed * 10 + 2).cuda()
    vc = inputs.randn_bf16((B, L, Hkv, D), seed * 10 + 3).cuda()
    win = wp.Window(D, base, alpha, g)
    k_pos = torch.arange(L, dtype=torch.int32).repeat(B, 1).cuda()
    out_p, lse_p = wp.decode_positions(q, kc, vc, kv_len, [n - 1 for n in kv_len], k_pos, win)
    out_d, lse_d = wp.decode(q, kc, vc, kv_len, win)
    assert wp.device_status() == wp.OK
    assert torch.equal(out_p, out_d) and torch.equal(lse_p, lse_d)


POS_CASES = [
    # D, g, alpha, base, B, Hq, Hkv, kv_len, mode
    (128, 1, 1.0, 5e5, 3, 24, 8, [1000, 1, 517], "evicted"),
    (64, 8, 1.0, 1e6, 2, 14, 2, [3000, 2999], "shuffled"),
    (128, 8, 1.0, 1e4, 2, 28, 4, [2000, 70], "future"),
    (64, 1, 2.0, 1e4, 4, 9, 3, [2048, 1, 2, 1999], "future"),
    (128, 1, 0.05, 1e4, 1, 12, 1, [4100], "shuffled"),
    (128, 1, float("inf"), 5e5, 2, 16, 1, [700, 64], "evicted"),
]


@pytest.mark.parametrize("case", POS_CASES, ids=[str(i) for i in range(len(POS_CASES))])
def test_positions_vs_oracle(cuda_dev, case):
    D, g, alpha, base, B, Hq, Hkv, kv_len, mode = case
    seed = len(str(case)) + 800
    L = max(kv_len)
    q = inputs.randn_bf16((B, Hq, D), seed * 10 + 1)
    kc = inputs.randn_bf16((B, L, Hkv, D), seed * 10 + 2)
    vc = inputs.randn_bf16((B, L, Hkv, D), seed * 10 + 3)
    q_pos, k_pos = inputs.key_positions(kv_len, seed, mode, span=3.0)
    win = wp.Window(D, base, alpha, g)
    out, lse = wp.decode_positions(q.cuda(), kc.cuda(), vc.cuda(), kv_len, q_pos, k_pos.cuda(), win)
    assert wp.device_status() == wp.OK
    o_ref, l_ref = _oracle_positions(q, kc, vc, kv_len, q_pos, k_pos, Hq=Hq, Hkv=Hkv, D=D,
                                     base=base, alpha=alpha, g=g, scale=1.0 / math.sqrt(D))
    check_rows(*_all_rows(out, lse, B, Hq), o_ref, l_ref, str(case))


def test_positions_all_keys_in_future_give_empty_rows(cuda_dev):
    D, B, Hq, Hkv, L = 64, 2, 4, 2, 300
    q = inputs.randn_bf16((B, Hq, D), 1).cuda()
    kc = inputs.randn_bf16((B, L, Hkv, D), 2).cuda()
    k_pos = torch.stack([torch.arange(1000, 1000 + L), torch.arange(L)]).to(torch.int32).cuda()
    out, lse = wp.decode_positions(q, kc, kc, [L, L], [999, L - 1], k_pos,
                                   wp.Window(D, 1e4, 1.0, 1))
    assert wp.device_status() == wp.OK
    assert (out[0].float() == 0).all() and torch.isneginf(lse[0]).all()
    assert torch.isfinite(lse[1]).all()


def test_negative_position_is_reported(cuda_dev):
    D, L = 64, 100
    q = inputs.randn_bf16((1, 2, D), 1).cuda()
    kc = inputs.randn_bf16((1, L, 1, D), 2).cuda()
    k_pos = torch.arange(L, dtype=torch.int32)
    k_pos[17] = -5
    wp.decode_positions(q, kc, kc, [L], [L - 1], k_pos[None].cuda(), wp.Window(D, 1e4, 1.0, 1))
    assert wp.device_status() == wp.EINDEX
    assert wp.device_status() == wp.OK      # read and cleared


PAGED_CASES = [
    # D, g, alpha, base, B, Hq, Hkv, kv_len, page_size
    (128, 1, 1.0, 5e5, 3, 24, 8, [1000, 1, 517], 16),
    (64, 8, 1.0, 1e6, 2, 14, 2, [3000, 2999], 8),
    (128, 8, 1.0, 1e7, 1, 28, 4, [5000], 64),
    (64, 1, 2.0, 1e4, 4, 9, 3, [2048, 1, 2, 1999], 32),
    (128, 1, 0.05, 1e4, 2, 12, 1, [4100, 900], 256),
    (128, 1, float("inf"), 5e5, 2, 16, 1, [700, 64], 16),
]


@pytest.mark.parametrize("case", PAGED_CASES, ids=[str(i) for i in range(len(PAGED_CASES))])
@pytest.mark.parametrize("positions", [False, True])
def test_paged_equals_gathered_and_oracle(cuda_dev, case, positions):
    D, g, alpha, base, B, Hq, Hkv, kv_len, page_size = case
    seed = len(str(case)) + 900 + positions
    L = max(kv_len)
    q = inputs.randn_bf16((B, Hq, D), seed * 10 + 1)
    kc = inputs.randn_bf16((B, L, Hkv, D), seed * 10 + 2)
    vc = inputs.randn_bf16((B, L, Hkv, D), seed * 10 + 3)
    table, num_pages = inputs.page_layout(kv_len, page_size, seed)
    kp = inputs.scatter_to_pages(kc, kv_len, table, page_size, num_pages)
    vp = inputs.scatter_to_pages(vc, kv_len, table, page_size, num_pages)
    win = wp.Window(D, base, alpha, g)
    q_pos, k_pos = inputs.key_positions(kv_len, seed, "shuffled") if positions else (None, None)
    qd = q.cuda()
    out, lse = wp.decode_paged(qd, kp.cuda(), vp.cuda(), table.cuda(), kv_len, win, q_pos=q_pos,
                               k_pos=k_pos.cuda() if positions else None)
    assert wp.device_status() == wp.OK
    # the gathered cache (NaN past each sequence's pages) through the contiguous call
    kg = inputs.gather_pages(kp, kv_len, table).cuda()
    vg = inputs.gather_pages(vp, kv_len, table).cuda()
    if positions:
        kpos_g = torch.full((B, kg.shape[1]), -1, dtype=torch.int32)
        kpos_g[:, :k_pos.shape[1]] = k_pos
        out_c, lse_c = wp.decode_positions(qd, kg, vg, kv_len, q_pos, kpos_g.cuda(), win)
    else:
        out_c, lse_c = wp.decode(qd, kg, vg, kv_len, win)
    assert wp.device_status() == wp.OK
    assert torch.equal(out, out_c) and torch.equal(lse, lse_c)
    if positions:
        o_ref, l_ref = _oracle_positions(q, kc, vc, kv_len, q_pos, k_pos, Hq=Hq, Hkv=Hkv, D=D,
                                         base=base, alpha=alpha, g=g, scale=1.0 / math.sqrt(D))
    else:
        o_ref, l_ref = oracle.decode_rows(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len,
                                          Hq=Hq, Hkv=Hkv, base=base, alpha=alpha, g=g,
                                          scale=1.0 / math.sqrt(D))
    check_rows(*_all_rows(out, lse, B, Hq), o_ref, l_ref, str(case))


def test_paged_bad_page_is_reported(cuda_dev):
    D, B, Hq, Hkv, page = 64, 1, 2, 1, 16
    kv_len = [100]
    table, num_pages = inputs.page_layout(kv_len, page, 3)
    kc = inputs.randn_bf16((B, 112, Hkv, D), 2)
    kp = inputs.scatter_to_pages(kc, kv_len, table, page, num_pages).cuda()
    q = inputs.randn_bf16((B, Hq, D), 1).cuda()
    bad = table.clone()
    bad[0, 3] = num_pages            # one past the pool
    wp.decode_paged(q, kp, kp, bad.cuda(), kv_len, wp.Window(D, 1e4, 1.0, 1))
    assert wp.device_status() == wp.EINDEX
    wp.decode_paged(q, kp, kp, table.cuda(), kv_len, wp.Window(D, 1e4, 1.0, 1))
    assert wp.device_status() == wp.OK


def test_paged_rejects_bad_args(cuda_dev):
    D = 64
    win = wp.Window(D, 1e4, 1.0, 1)
    q = inputs.randn_bf16((1, 2, D), 1).cuda()
    pool = torch.zeros((4, 24, 1, D), dtype=torch.bfloat16, device="cuda")
    table = torch.zeros((1, 4), dtype=torch.int32, device="cuda")
    with pytest.raises(wp.WpattnError) as e:            # page size 24
        wp.decode_paged(q, pool, pool, table, [50], win)
    assert e.value.code == wp.EUNSUPPORTED
    pool = torch.zeros((4, 16, 1, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wp.WpattnError) as e:            # kv_len beyond the table's reach
        wp.decode_paged(q, pool, pool, table, [65], win)
    assert e.value.code == wp.EINVAL
    with pytest.raises(wp.WpattnError) as e:            # q_pos without k_pos
        wp.decode_paged(q, pool, pool, table, [50], win, q_pos=[49])
    assert e.value.code == wp.EINVAL


@pytest.mark.parametrize("name,n_rows,page_size", [("llama3.2-3b-decode-128k", 24, 16),
                                                    ("qwen2.5-7b-1m-decode", 14, 64)])
def test_paged_positions_full_size(cuda_dev, name, n_rows, page_size):
    """Full-size caches, paged and with evicted positions, sampled rows vs the oracle."""
    w = inputs.WORKLOADS[name]
    q, kc, vc, kv_len = inputs.decode_inputs(w, seed=0, device=torch.device("cuda:0"))
    kv_len = [int(x) for x in kv_len]
    table, num_pages = inputs.page_layout(kv_len, page_size, 5)
    kp = inputs.scatter_to_pages(kc, kv_len, table, page_size, num_pages)
    vp = inputs.scatter_to_pages(vc, kv_len, table, page_size, num_pages)
    q_pos, k_pos = inputs.key_positions(kv_len, 6, "evicted")
    win = wp.Window(w.D, w.base, w.alpha, w.g)
    out, lse = wp.decode_paged(q, kp, vp, table.cuda(), kv_len, win, q_pos=q_pos,
                               k_pos=k_pos.cuda(), scale=w.scale)
    assert wp.device_status() == wp.OK
    del kp, vp
    rng = np.random.default_rng(12)
    rows = sorted({(int(rng.integers(0, w.B)), int(rng.integers(0, w.Hq))) for _ in range(n_rows)})
    o_ref, l_ref = oracle.decode_positions(inputs.bits(q), inputs.bits(kc), inputs.bits(vc),
                                           kv_len, q_pos, k_pos.numpy().astype(np.int64), Hq=w.Hq,
                                           Hkv=w.Hkv, base=w.base, alpha=w.alpha, g=w.g,
                                           scale=w.scale, rows=rows)
    oc, lc = out.float().cpu(), lse.cpu()
    check_rows(np.stack([oc[b, h].numpy() for (b, h) in rows]),
               np.array([float(lc[b, h]) for (b, h) in rows]), o_ref, l_ref, name)
