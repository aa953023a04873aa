"""Pair-major K cache: the layout conversion (bit-exact against a plain index
permutation on the host) and decode from the slabs (against the oracle, and
bitwise against decode from the [B, L, Hkv, D] cache, which runs the same
arithmetic in the same order), through the C ABI."""
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


def _slabs_reference(k_bits):
    """[B, L, Hkv, D] uint16 -> [B, Hkv, D/16, L, 16]: slab g = dims 8g..8g+7, then D/2+8g..D/2+8g+7."""
    B, L, Hkv, D = k_bits.shape
    P, NG = D // 2, D // 16
    out = np.empty((B, Hkv, NG, L, 16), dtype=k_bits.dtype)
    for g in range(NG):
        out[:, :, g, :, :8] = k_bits[:, :, :, 8 * g:8 * g + 8].transpose(0, 2, 1, 3)
        out[:, :, g, :, 8:] = k_bits[:, :, :, P + 8 * g:P + 8 * g + 8].transpose(0, 2, 1, 3)
    return out


@pytest.mark.parametrize("shape", [(1, 1, 1, 64), (2, 77, 3, 128), (3, 1000, 2, 64), (1, 4096, 8, 128)])
def test_kcache_to_pairmajor_bit_exact(cuda_dev, shape):
    k = inputs.randn_bf16(shape, 901 + shape[1])
    slabs = wp.kcache_to_pairmajor(k.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(inputs.bits(slabs.cpu()), _slabs_reference(inputs.bits(k)))


def test_kcache_to_pairmajor_rejects_bad_args(cuda_dev):
    k = inputs.randn_bf16((1, 8, 1, 96), 3).cuda()
    with pytest.raises(wp.WpattnError) as e:
        wp.kcache_to_pairmajor(k, out=torch.empty((1, 1, 6, 8, 16), dtype=torch.bfloat16, device="cuda"))
    assert e.value.code == wp.EUNSUPPORTED


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_decode_pairmajor_all_rows(cuda_dev, case):
    D, g, alpha, base, B, Hq, Hkv, L, kv_len = case
    seed = len(str(case)) + 500
    q = inputs.randn_bf16((B, Hq, D), seed * 10 + 1)
    kc = inputs.randn_bf16((B, L, Hkv, D), seed * 10 + 2)
    vc = inputs.randn_bf16((B, L, Hkv, D), seed * 10 + 3)
    win = wp.Window(D, base, alpha, g)
    qd, kd, vd = q.cuda(), kc.cuda(), vc.cuda()
    out_pm, lse_pm = wp.decode_pairmajor(qd, wp.kcache_to_pairmajor(kd), vd, kv_len, win)
    out_st, lse_st = wp.decode(qd, kd, vd, kv_len, win)
    assert wp.device_status() == wp.OK
    # same arithmetic in the same order: identical bits
    assert torch.equal(out_pm, out_st) and torch.equal(lse_pm, lse_st)
    rows = [(b, h) for b in range(B) for h in range(Hq)]
    o_ref, l_ref = oracle.decode_rows(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len,
                                      Hq=Hq, Hkv=Hkv, base=base, alpha=alpha, g=g,
                                      scale=1.0 / math.sqrt(D), rows=rows)
    oc, lc = out_pm.float().cpu(), lse_pm.cpu()
    check_rows(np.stack([oc[b, h].numpy() for (b, h) in rows]),
               np.array([float(lc[b, h]) for (b, h) in rows]), o_ref, l_ref, str(case))


@pytest.mark.parametrize("name,n_rows", [("llama3.2-3b-decode-128k", 24),
                                         ("qwen2.5-7b-1m-decode", 14)])
def test_decode_pairmajor_full_size(cuda_dev, name, n_rows):
    w = inputs.WORKLOADS[name]
    dev = torch.device("cuda:0")
    q, kc, vc, kv_len = inputs.decode_inputs(w, seed=0, device=dev)
    kv_len = [int(x) for x in kv_len]
    win = wp.Window(w.D, w.base, w.alpha, w.g)
    slabs = wp.kcache_to_pairmajor(kc)
    out, lse = wp.decode_pairmajor(q, slabs, vc, kv_len, win, scale=w.scale)
    assert wp.device_status() == wp.OK
    rng = np.random.default_rng(11)
    rows = sorted({(int(rng.integers(0, w.B)), int(rng.integers(0, w.Hq))) for _ in range(n_rows)})
    o_ref, l_ref = oracle.decode_rows(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len,
                                      Hq=w.Hq, Hkv=w.Hkv, base=w.base, alpha=w.alpha, g=w.g,
                                      scale=w.scale, rows=rows)
    oc, lc = out.float().cpu(), lse.cpu()
    check_rows(np.stack([oc[b, h].numpy() for (b, h) in rows]),
               np.array([float(lc[b, h]) for (b, h) in rows]), o_ref, l_ref, name)
