"""Decode with the cache split by length, through the C ABI on one GPU: the
shards of 2 to 4 ranks are attended one after the other (no rank waits on
another) and merged with merge_lse; the result is compared with the oracle's
decode over the whole cache.  Also the merge kernel alone against a float64
merge, and the argument checks of the shard call."""
import math

import numpy as np
import pytest
import torch

import oracle
import rope_wavelength_sparsity_b200 as wp
from rope_wavelength_sparsity_b200 import distributed as wd
from rope_wavelength_sparsity_b200 import inputs

from _parity import check_rows

pytestmark = pytest.mark.gpu

CASES = [
    # D, g, alpha, base, B, Hq, Hkv, shard_len, world, kv_len
    (128, 1, 1.0, 5e5, 3, 24, 8, 512, 2, [1024, 300, 700]),
    (64, 8, 1.0, 1e6, 2, 14, 2, 1000, 3, [3000, 2001]),
    (128, 8, 1.0, 1e7, 1, 28, 4, 1024, 4, [4096]),
    (128, 1, float("inf"), 5e5, 2, 16, 1, 256, 4, [1000, 64]),
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_shards_merged_vs_oracle(cuda_dev, case):
    D, g, alpha, base, B, Hq, Hkv, shard, world, kv_len = case
    seed = len(str(case)) + 1100
    L = shard * world
    q = inputs.randn_bf16((B, Hq, D), seed * 10 + 1)
    kc = inputs.randn_bf16((B, L, Hkv, D), seed * 10 + 2)
    vc = inputs.randn_bf16((B, L, Hkv, D), seed * 10 + 3)
    win = wp.Window(D, base, alpha, g)
    qd = q.cuda()
    outs, lses = [], []
    for r in range(world):
        k_pos0, n = wd.shard_keys(kv_len, r, shard)
        ks = kc[:, r * shard:(r + 1) * shard].contiguous().cuda()
        vs = vc[:, r * shard:(r + 1) * shard].contiguous().cuda()
        o, l = wp.decode_shard(qd, ks, vs, n, [x - 1 for x in kv_len], k_pos0, win)
        outs.append(o)
        lses.append(l)
    out, lse = wp.merge_lse(torch.stack(outs), torch.stack(lses))
    assert wp.device_status() == wp.OK
    rows = [(b, h) for b in range(B) for h in range(Hq)]
    o_ref, l_ref = oracle.decode_rows(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len,
                                      Hq=Hq, Hkv=Hkv, base=base, alpha=alpha, g=g,
                                      scale=1.0 / math.sqrt(D), rows=rows)
    oc, lc = out.float().cpu(), lse.cpu()
    check_rows(np.stack([oc[b, h].numpy() for (b, h) in rows]),
               np.array([float(lc[b, h]) for (b, h) in rows]), o_ref, l_ref, str(case))
    # a shard that holds no key of a sequence reports it empty
    if any(x <= (world - 1) * shard for x in kv_len):
        last = torch.stack(lses)[world - 1].cpu()
        for b, x in enumerate(kv_len):
            if x <= (world - 1) * shard:
                assert torch.isneginf(last[b]).all()


@pytest.mark.parametrize("D", [64, 128])
def test_merge_lse_vs_float64(cuda_dev, D):
    R, rows = 5, 300
    g = torch.Generator().manual_seed(D)
    outs = torch.randn((R, rows, D), generator=g).to(torch.bfloat16)
    lses = torch.randn((R, rows), generator=g) * 4
    lses[1, :50] = -math.inf                     # empty parts
    lses[:, 7] = -math.inf                       # a row with no part at all
    out, lse = wp.merge_lse(outs.cuda(), lses.cuda())
    torch.cuda.synchronize()
    o = outs.double().numpy()
    l = lses.double().numpy()
    M = l.max(axis=0)
    with np.errstate(invalid="ignore"):
        w = np.where(np.isneginf(l), 0.0, np.exp(l - M))
    W = w.sum(axis=0)
    ok = W > 0
    want = np.zeros((rows, D))
    want[ok] = (w[:, ok, None] * o[:, ok]).sum(axis=0) / W[ok, None]
    np.testing.assert_allclose(out.float().cpu().numpy(), want, atol=8e-3, rtol=8e-3)
    np.testing.assert_allclose(lse.cpu().numpy()[ok], (M + np.log(np.where(ok, W, 1.0)))[ok],
                               atol=1e-5)
    assert math.isinf(float(lse[7])) and (out[7].float() == 0).all()


def test_decode_shard_rejects_keys_after_the_query(cuda_dev):
    D = 64
    q = inputs.randn_bf16((1, 2, D), 1).cuda()
    ks = inputs.randn_bf16((1, 100, 1, D), 2).cuda()
    with pytest.raises(wp.WpattnError) as e:                # keys 50..149, query at 120
        wp.decode_shard(q, ks, ks, [100], [120], [50], wp.Window(D, 1e4, 1.0, 1))
    assert e.value.code == wp.EINVAL
