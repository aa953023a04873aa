"""Prefill with work items' key ranges split into parts (each part's rows
normalised over its own keys, merged by their log-sum-exp): every output row
against the oracle for forced split counts, including parts that hold no key
of a query block (causal rows, ragged key tails, more parts than key tiles),
rows that see no key at all, the library's own plan on chunks at a long
context (all items split; only the last partial wave split), and the
workspace checks of the C entry point."""
import ctypes
import math

import numpy as np
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


SPLIT_CASES = [
    # D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q_pos0, k_pos0, kv_splits
    (128, 8, 1.0, 1e7, 1, 4, 1, 300, 1500, 1200, 0, 2),   # chunk at the end of the keys
    (128, 8, 1.0, 1e7, 1, 4, 1, 300, 1500, 1200, 0, 3),   # parts of 4, 4 and 4 tiles
    (64, 8, 1.0, 1e6, 2, 7, 1, 257, 1000, 743, 0, 5),     # GQA 7, batch 2, ragged last tile
    (128, 1, 1.0, 5e5, 1, 3, 1, 520, 520, 0, 0, 2),       # causal: block 0 sees only part 0
    (64, 1, 0.3, 1e4, 1, 2, 2, 450, 450, 0, 0, 4),        # partial k-steps, g = 1
    (128, 1, 2.0, 5e5, 1, 2, 1, 200, 300, 100, 0, 7),     # more parts than key tiles (3)
    (64, 1, 1.0, 1e4, 1, 2, 1, 200, 150, 0, 60, 2),       # first 60 rows see no key
    (64, 8, float("inf"), 1e4, 1, 2, 1, 260, 900, 640, 0, 3),  # window off
]


@pytest.mark.parametrize("case", SPLIT_CASES, ids=[str(i) for i in range(len(SPLIT_CASES))])
def test_prefill_split_all_rows(cuda_dev, case):
    D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q0, k0, S = case
    q, k, v = _qkv(B, Nq, Nk, Hq, Hkv, D, seed=len(str(case)) + 700)
    prefill_parity(q, k, v, Hq=Hq, Hkv=Hkv, D=D, base=base, alpha=alpha, g=g, q_pos0=q0,
                   k_pos0=k0, kv_splits=S, what=str(case))


def test_prefill_split_close_to_unsplit(cuda_dev):
    """Split and unsplit differ only by the rounding order of the merge."""
    q, k, v = _qkv(1, 256, 4096, 4, 2, 128, seed=41)
    win = wp.Window(128, 1e7, 1.0, 8)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = wp.prefill(qd, kd, vd, win, q_pos0=3840, kv_splits=1)
    o4, l4 = wp.prefill(qd, kd, vd, win, q_pos0=3840, kv_splits=4)
    torch.cuda.synchronize()
    assert wp.device_status() == wp.OK
    assert (o1.float() - o4.float()).abs().max().item() <= 1e-2
    assert (l1 - l4).abs().max().item() <= 1e-4


def test_prefill_split_library_plan_all_items(cuda_dev):
    """A 256-row chunk at the end of 64K keys on 20 heads: 20 equal items fill a
    seventh of a wave, so the library splits all of them (7 parts on 148 SMs),
    and the merged rows match the oracle."""
    B, Hq, Hkv, D, Nq, Nk = 1, 20, 4, 128, 256, 65536
    q0 = Nk - Nq
    main, n_split, parts = wp.prefill_split_plan(B, Nq, Nk, Hq, q0, 0)
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert (main, n_split, parts) == (0, 20, 7)
    assert n_split > 0 and parts >= 2
    q, k, v = _qkv(B, Nq, Nk, Hq, Hkv, D, seed=43)
    rows = [(0, h, t) for h in (0, 7, 19) for t in (0, 1, 127, 128, 255)]
    prefill_parity(q, k, v, Hq=Hq, Hkv=Hkv, D=D, base=1e7, alpha=1.0, g=8, q_pos0=q0, rows=rows,
                   what="library plan, all items")


def test_prefill_split_library_plan_last_wave(cuda_dev):
    """150 equal items on 148 SMs: the first 148 run unsplit, the last 2 (heads
    148 and 149) in 8 parts each; rows of both kinds match the oracle."""
    B, Hq, Hkv, D, Nq, Nk = 1, 150, 2, 64, 256, 65536
    q0 = Nk - Nq
    plan = wp.prefill_split_plan(B, Nq, Nk, Hq, q0, 0)
    if torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert plan == (148, 2, 8)
    q, k, v = _qkv(B, Nq, Nk, Hq, Hkv, D, seed=44)
    rows = [(0, h, t) for h in (0, 75, 147, 148, 149) for t in (0, 127, 128, 200, 255)]
    prefill_parity(q, k, v, Hq=Hq, Hkv=Hkv, D=D, base=1e6, alpha=1.0, g=8, q_pos0=q0, rows=rows,
                   what="library plan, last wave")


def test_prefill_split_unsplit_items_bitwise(cuda_dev):
    """Under the library's last-wave plan the unsplit items run the plain kernel: their rows
    equal an unsplit call bit for bit; the split items' rows agree within the bar."""
    B, Hq, Hkv, D, Nq, Nk = 1, 150, 2, 64, 256, 65536
    q0 = Nk - Nq
    main, n_split, parts = wp.prefill_split_plan(B, Nq, Nk, Hq, q0, 0)
    if n_split == 0:
        pytest.skip("this device's plan splits nothing for the shape")
    q, k, v = _qkv(B, Nq, Nk, Hq, Hkv, D, seed=46)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    win = wp.Window(D, 1e6, 1.0, 8)
    o_s, l_s = wp.prefill(qd, kd, vd, win, q_pos0=q0)
    o_1, l_1 = wp.prefill(qd, kd, vd, win, q_pos0=q0, kv_splits=1)
    torch.cuda.synchronize()
    assert wp.device_status() == wp.OK
    # with one query block per head (Nq = 256) item i is head i
    assert torch.equal(o_s[:, :, :main], o_1[:, :, :main])
    assert torch.equal(l_s[:, :main], l_1[:, :main])
    assert (o_s[:, :, main:].float() - o_1[:, :, main:].float()).abs().max().item() <= 1e-2
    assert (l_s[:, main:] - l_1[:, main:]).abs().max().item() <= 1e-4


def test_prefill_split_workspace_checks(cuda_dev):
    q, k, v = _qkv(1, 256, 1024, 2, 1, 64, seed=45)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out = torch.empty_like(qd)
    win = wp.Window(64, 1e4, 1.0, 1)
    need = wp.prefill_split_workspace_size(1, 256, 1024, 2, 64, 768, 0, 4)
    assert need == 4 * 2 * 256 * 65 * 4
    L = wp.lib()

    def call(ws, nbytes, S=4):
        return L.wpattn_prefill_split(ctypes.byref(win._c()), ctypes.c_void_p(qd.data_ptr()),
                                      ctypes.c_void_p(kd.data_ptr()), ctypes.c_void_p(vd.data_ptr()),
                                      ctypes.c_void_p(out.data_ptr()), None, 1, 256, 1024, 2, 1, 768,
                                      0, 0.0, S, ws, nbytes, None)

    ws = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
    assert call(ctypes.c_void_p(ws.data_ptr()), need - 1) == wp.EWORKSPACE
    assert call(None, need) == wp.EINVAL
    assert call(ctypes.c_void_p(ws.data_ptr() + 16), need) == wp.EINVAL   # not 256-byte aligned
    assert call(ctypes.c_void_p(ws.data_ptr()), need, S=-1) == wp.EINVAL
    assert call(ctypes.c_void_p(ws.data_ptr()), need) == wp.OK
    torch.cuda.synchronize()
    assert wp.device_status() == wp.OK
