"""Shared helpers for the GPU parity tests: run the CUDA path through the
C ABI, run the oracle on the same bf16 bytes, compare element by element."""
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
import rope_wavelength_sparsity_b200 as wp
from rope_wavelength_sparsity_b200 import inputs

# tolerances of the parity bar (out in bf16 units of the output, LSE in nats)
ATOL_OUT = 1e-2
ATOL_LSE = 2e-3


def oracle_rows_threaded(q_bits, k_bits, v_bits, rows, **kw):
    """oracle.attention_rows over many rows, split across host threads (the oracle's
    C code runs outside the GIL; each call computes its rows independently)."""
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    n_thr = max(1, min(len(rows), len(os.sched_getaffinity(0))))
    chunks = [c for c in np.array_split(rows, n_thr) if len(c)]
    with ThreadPoolExecutor(max_workers=len(chunks)) as ex:
        parts = list(ex.map(lambda c: oracle.attention_rows(q_bits, k_bits, v_bits, rows=c, **kw),
                            chunks))
    return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts])


def check_rows(o_gpu, l_gpu, o_ref, l_ref, what):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    l_gpu = np.asarray(l_gpu, dtype=np.float64)
    empty = np.isneginf(l_ref)
    assert np.array_equal(np.isneginf(l_gpu), empty), f"{what}: empty-row mismatch"
    if empty.any():
        assert (o_gpu[empty] == 0).all(), f"{what}: empty rows must be 0"
    ok = ~empty
    with np.errstate(invalid="ignore"):  # empty rows: -inf - -inf, masked out below
        err_o = np.where(ok[:, None], np.abs(o_gpu - o_ref), 0.0).max(axis=1)
        err_l = np.where(ok, np.abs(l_gpu - l_ref), 0.0)
    d_out, d_lse = float(err_o.max()), float(err_l.max())
    bad = np.nonzero((err_o > ATOL_OUT) | (err_l > ATOL_LSE))[0]
    assert d_out <= ATOL_OUT and d_lse <= ATOL_LSE, (
        f"{what}: max|dout|={d_out:.3e} max|dlse|={d_lse:.3e}; {len(bad)} of {len(ok)} rows "
        f"out of tolerance, first: {bad[:12].tolist()}")
    return d_out, d_lse


def prefill_parity(q, k, v, *, Hq, Hkv, D, base, alpha, g, q_pos0=0, k_pos0=0, rows=None,
                   scale=None, what="", kv_splits=None):
    """q, k, v: bf16 tensors (any device).  Returns (max dout, max dlse).
    kv_splits: passed to wp.prefill (None = the library's choice)."""
    dev = torch.device("cuda:0")
    B, Nq = q.shape[0], q.shape[1]
    scale = scale or 1.0 / math.sqrt(D)
    win = wp.Window(D, base, alpha, g)
    out, lse = wp.prefill(q.to(dev), k.to(dev), v.to(dev), win, q_pos0=q_pos0, k_pos0=k_pos0,
                          scale=scale, kv_splits=kv_splits)
    assert wp.device_status() == wp.OK
    if rows is None:
        rows = [(b, h, t) for b in range(B) for h in range(Hq) for t in range(Nq)]
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    o_ref, l_ref = oracle.attention_rows(inputs.bits(q), inputs.bits(k), inputs.bits(v), Hq=Hq,
                                         Hkv=Hkv, q_pos0=q_pos0, k_pos0=k_pos0, base=base,
                                         alpha=alpha, g=g, scale=scale, rows=rows)
    bi, hi, ti = (torch.as_tensor(rows[:, i]) for i in range(3))
    o_gpu = out.float().cpu()[bi, ti, hi].numpy()
    l_gpu = lse.cpu()[bi, hi, ti].numpy()
    return check_rows(o_gpu, l_gpu, o_ref, l_ref, what)


def decode_parity(q, kc, vc, kv_len, *, Hq, Hkv, D, base, alpha, g, rows=None, scale=None,
                  what=""):
    dev = torch.device("cuda:0")
    B = q.shape[0]
    scale = scale or 1.0 / math.sqrt(D)
    win = wp.Window(D, base, alpha, g)
    kv_len = [int(x) for x in kv_len]
    out, lse = wp.decode(q.to(dev), kc.to(dev), vc.to(dev), kv_len, win, scale=scale)
    assert wp.device_status() == wp.OK
    if rows is None:
        rows = [(b, h) for b in range(B) for h in range(Hq)]
    o_ref, l_ref = oracle.decode_rows(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len,
                                      Hq=Hq, Hkv=Hkv, base=base, alpha=alpha, g=g, scale=scale,
                                      rows=rows)
    oc, lc = out.float().cpu(), lse.cpu()
    o_gpu = np.stack([oc[b, h].numpy() for (b, h) in rows])
    l_gpu = np.array([float(lc[b, h]) for (b, h) in rows])
    return check_rows(o_gpu, l_gpu, o_ref, l_ref, what)
