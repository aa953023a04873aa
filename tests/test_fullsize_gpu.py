"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times (the same public calls, same shapes, windows and inputs).

Inputs are drawn on the GPU from the seeded generators and copied to the
host for the oracle, which recomputes sampled output rows one by one: the
first and last rows, rows on both sides of a 128-row tile boundary, rows in
the middle of the sequence, and the planted-key rows of the Llama-shaped
workloads (which must also put > 0.99 of their weight on the planted key).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import rope_wavelength_sparsity_b200 as wp
from rope_wavelength_sparsity_b200 import inputs

from _parity import check_rows, oracle_rows_threaded

pytestmark = pytest.mark.gpu


def _prefill_rows(w, planted, per_head):
    rows = []
    for h in range(w.Hq):
        for t in per_head:
            if 0 <= t < w.Nq:
                rows.append((0, h, t))
    rows += [(b, hq, t) for (b, hq, t, _, _) in planted]
    return rows


def _run_prefill(name, per_head):
    w = inputs.WORKLOADS[name]
    dev = torch.device("cuda:0")
    q, k, v, planted = inputs.prefill_inputs(w, seed=0, device=dev)
    win = wp.Window(w.D, w.base, w.alpha, w.g)
    out, lse = wp.prefill(q, k, v, win, q_pos0=w.q_pos0, k_pos0=w.k_pos0, scale=w.scale)
    assert wp.device_status() == wp.OK
    rows = np.asarray(_prefill_rows(w, planted, per_head), dtype=np.int64)
    qb, kb, vb = inputs.bits(q), inputs.bits(k), inputs.bits(v)
    o_ref, l_ref = oracle_rows_threaded(qb, kb, vb, rows, Hq=w.Hq, Hkv=w.Hkv, q_pos0=w.q_pos0,
                                        k_pos0=w.k_pos0, base=w.base, alpha=w.alpha, g=w.g,
                                        scale=w.scale)
    oc = out.float().cpu()
    lc = lse.cpu()
    o_gpu = np.stack([oc[b, t, h].numpy() for (b, h, t) in rows])
    l_gpu = np.array([float(lc[b, h, t]) for (b, h, t) in rows])
    check_rows(o_gpu, l_gpu, o_ref, l_ref, name)
    for (b, hq, t, kvh, j) in planted:
        s = oracle.scores(qb[b, t, hq], kb[b, :, kvh], q_pos=w.q_pos0 + t, k_pos0=w.k_pos0,
                          base=w.base, alpha=w.alpha, g=w.g)
        n = int(np.nonzero((rows[:, 0] == b) & (rows[:, 1] == hq) & (rows[:, 2] == t))[0][0])
        weight = math.exp(w.scale * s[j] - l_ref[n])
        assert weight > 0.99, (name, kvh, j, weight)          # reachable through low-frequency pairs
        assert abs(float(lc[b, hq, t]) - l_ref[n]) <= 2e-3
    return w


BOUNDARY = [0, 1, 127, 128, 129, 255, 256, 4095, 4096]


def test_qwen_0_5b_32k_prefill(cuda_dev):
    _run_prefill("qwen2.5-0.5b-32k", BOUNDARY + [16383, 16384, 30000, 32767])


@pytest.mark.parametrize("name", ["llama3.2-3b-128k-a1", "llama3.2-3b-128k-a2"])
def test_llama_3b_128k_prefill(cuda_dev, name):
    _run_prefill(name, [0, 128, 65535, 65536, 131071])


def test_qwen_7b_1m_last_chunk_prefill(cuda_dev):
    # both ends of the chunk, both sides of 128- and 256-row tile boundaries, the middle
    _run_prefill("qwen2.5-7b-1m-prefill", [0, 1, 127, 128, 255, 256, 8191, 8192, 16256, 16383])


@pytest.mark.parametrize("name,n_rows", [("llama3.2-3b-decode-128k", 32),
                                         ("qwen2.5-7b-1m-decode", 28)])
def test_decode_full_size(cuda_dev, name, n_rows):
    w = inputs.WORKLOADS[name]
    dev = torch.device("cuda:0")
    q, kc, vc, kv_len = inputs.decode_inputs(w, seed=0, device=dev)
    kv_len = [int(x) for x in kv_len]
    win = wp.Window(w.D, w.base, w.alpha, w.g)
    out, lse = wp.decode(q, kc, vc, kv_len, win, scale=w.scale)
    assert wp.device_status() == wp.OK
    rng = np.random.default_rng(5)
    rows = sorted({(int(rng.integers(0, w.B)), int(rng.integers(0, w.Hq))) for _ in range(n_rows)})
    o_ref, l_ref = oracle.decode_rows(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len,
                                      Hq=w.Hq, Hkv=w.Hkv, base=w.base, alpha=w.alpha, g=w.g,
                                      scale=w.scale, rows=rows)
    oc, lc = out.float().cpu(), lse.cpu()
    check_rows(np.stack([oc[b, h].numpy() for (b, h) in rows]),
               np.array([float(lc[b, h]) for (b, h) in rows]), o_ref, l_ref, name)
