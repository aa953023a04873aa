"""Host-side checks of the C-ABI library (no GPU needed).

- the shared library loads and exports every function include/wpattn.h declares;
- the planner's thresholds and closed-form pruned-term counts equal the
  oracle's bit for bit (the oracle derives them independently);
- argument errors come back as status codes before any device work.
"""
import ctypes
import math
import os
import re

import pytest

import oracle
import rope_wavelength_sparsity_b200 as wp
from rope_wavelength_sparsity_b200 import build, inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(wpattn_\w+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert {"wpattn_prefill", "wpattn_decode", "wpattn_pruned_fraction"} <= set(names)
    L = ctypes.CDLL(wp.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    assert wp.version().count(".") == 2


WINDOWS = [
    (64, 1e4, 1.0, 1), (64, 1e6, 1.0, 8), (128, 5e5, 1.0, 1), (128, 5e5, 2.0, 1),
    (128, 1e7, 1.0, 8), (128, 5e5, 0.37, 8), (64, 1e4, float("inf"), 1), (4, 100.0, 1.0, 1),
    (16, 10.0, 3.3, 8), (256, 1e4, 1.0, 1),
]


@pytest.mark.parametrize("D,base,alpha,g", WINDOWS)
def test_thresholds_match_oracle(D, base, alpha, g):
    T_lib = wp.thresholds(wp.Window(D, base, alpha, g))
    T_or, _ = oracle.thresholds(D, base, alpha, g)
    assert T_lib == T_or.tolist()


@pytest.mark.parametrize("D,base,alpha,g", WINDOWS)
def test_closed_form_count_matches_oracle_small(D, base, alpha, g):
    w = wp.Window(D, base, alpha, g)
    for (Nq, Nk, q0, k0) in [(1, 1, 0, 0), (37, 37, 0, 0), (50, 130, 80, 0), (64, 20, 10, 30),
                             (5, 300, 299, 0), (40, 40, 0, 50), (0, 10, 0, 0), (10, 0, 0, 0),
                             (129, 1000, 871, 0), (300, 300, 7, 0)]:
        pr, tot, fr = wp.pruned_fraction(w, Nq, Nk, q0, k0)
        assert (pr, tot) == oracle.count_bruteforce(D, base, alpha, g, Nq, Nk, q0, k0)
        assert fr == (pr / tot if tot else 0.0)


@pytest.mark.parametrize("name", list(inputs.WORKLOADS))
def test_closed_form_count_matches_oracle_workloads(name):
    w = inputs.WORKLOADS[name]
    win = wp.Window(w.D, w.base, w.alpha, w.g)
    if w.kind == "prefill":
        args = (w.Nq, w.Nk, w.q_pos0, w.k_pos0)
    else:
        args = (1, w.Nk, w.Nk - 1, 0)
    pr, tot, _ = wp.pruned_fraction(win, *args)
    assert (pr, tot) == oracle.count_rows(w.D, w.base, w.alpha, w.g, *args)


def test_pruned_fraction_in_pages_range_for_group_reading():
    """ATFlash Abstract: 37-48 % pruned within native context (Qwen2.5-0.5B,
    Llama-3.2-3B) and 57 % at 1M (Qwen2.5-7B-1M, full 1M x 1M causal square).  Our g = 8 reading (group
    keeps its longest wavelength) at alpha = 2 lands in those ranges; this is
    a consistency check of the reading, not a pin of an exact number."""
    _, _, f = wp.pruned_fraction(wp.Window(64, 1e6, 2.0, 8), 32768, 32768)
    assert 0.37 <= f <= 0.48
    _, _, f = wp.pruned_fraction(wp.Window(128, 1e7, 2.0, 8), 1048576, 1048576)
    assert abs(f - 0.57) < 0.01


def test_argument_errors_are_status_codes():
    L = wp.lib()
    bad = [wp.Window(63, 1e4, 1.0, 1), wp.Window(64, 1.0, 1.0, 1), wp.Window(64, 1e4, 0.0, 1),
           wp.Window(64, 1e4, float("nan"), 1), wp.Window(64, 1e4, 1.0, 4),
           wp.Window(24, 1e4, 1.0, 8)]
    for w in bad:
        rc = L.wpattn_prefill(ctypes.byref(w._c()), None, None, None, None, None, 1, 1, 1, 1, 1,
                              0, 0, 0.0, None)
        assert rc == wp.EINVAL, w
        assert L.wpattn_decode_workspace_size(ctypes.byref(w._c()), 1, 1, 1, 10) == 0
    w = wp.Window(64, 1e4, 1.0, 1)
    # GQA mismatch, null tensors, unsupported head dim
    assert L.wpattn_prefill(ctypes.byref(w._c()), None, None, None, None, None, 1, 4, 4, 3, 2, 0, 0,
                            0.0, None) == wp.EINVAL
    assert L.wpattn_prefill(ctypes.byref(w._c()), None, None, None, None, None, 1, 4, 4, 2, 2, 0, 0,
                            0.0, None) == wp.EINVAL
    w96 = wp.Window(96, 1e4, 1.0, 1)
    assert L.wpattn_prefill(ctypes.byref(w96._c()), None, None, None, None, None, 1, 4, 4, 2, 2, 0,
                            0, 0.0, None) == wp.EUNSUPPORTED
    # empty problems are no-ops
    assert L.wpattn_prefill(ctypes.byref(w._c()), None, None, None, None, None, 0, 4, 4, 2, 2, 0, 0,
                            0.0, None) == wp.OK
    kvl = (ctypes.c_int32 * 1)(0)
    assert L.wpattn_decode(ctypes.byref(w._c()), ctypes.c_void_p(16), ctypes.c_void_p(16),
                           ctypes.c_void_p(16), kvl, 8, 1, 2, 2, 0.0, ctypes.c_void_p(16), None,
                           None, 0, None) == wp.EINVAL   # kv_len 0
    # the fused q and k rotation: bad sizes, base, head dim and positions are
    # refused before any launch; nothing to rotate is a no-op
    v16 = ctypes.c_void_p(16)
    assert L.wpattn_rope_qk(v16, v16, v16, v16, -1, 4, 4, 2, 2, 64, 0, 0, 1e4, None) == wp.EINVAL
    assert L.wpattn_rope_qk(v16, v16, v16, v16, 1, 4, 4, 2, 2, 64, 0, 0, 1.0, None) == wp.EINVAL
    assert L.wpattn_rope_qk(v16, v16, v16, v16, 1, 4, 4, 2, 2, 96, 0, 0, 1e4, None) == wp.EUNSUPPORTED
    assert L.wpattn_rope_qk(v16, v16, v16, v16, 1, 4, 4, 2, 2, 64, -1, 0, 1e4, None) == wp.EINVAL
    assert L.wpattn_rope_qk(v16, v16, v16, v16, 1, 4, 4, 2, 2, 64, 0, 2**41, 1e4, None) == wp.EINVAL
    assert L.wpattn_rope_qk(None, None, None, None, 1, 4, 0, 2, 2, 64, 0, 0, 1e4, None) == wp.EINVAL
    assert L.wpattn_rope_qk(None, None, None, None, 1, 0, 0, 2, 2, 64, 0, 0, 1e4, None) == wp.OK
    assert wp.lib().wpattn_strerror(wp.EWORKSPACE).decode() != "unknown status code"


def test_prefill_split_plan():
    """The library's key-range split: only for items of equal work (a chunk far into a
    long context), and only the items of the grid's last partial wave."""
    plan = wp.prefill_split_plan
    # 1M-key chunk, 28 heads: 1792 items = 12 waves of 148 + 16; the 16 go in 8 parts
    assert plan(1, 16384, 1048576, 28, 1032192, 0, 0, 148) == (1776, 16, 8)
    # causal self-attention (unequal items), or a grid of whole waves: nothing split
    assert plan(1, 131072, 131072, 24, 0, 0, 0, 148) == (12288, 0, 1)
    assert plan(1, 32768, 32768, 14, 0, 0, 0, 148) == (1792, 0, 1)
    assert plan(1, 256, 1048576, 148, 1048320, 0, 0, 148) == (148, 0, 1)
    # 20 items on 148 SMs: all of them in 7 parts
    assert plan(1, 256, 65536, 20, 65280, 0, 0, 148) == (0, 20, 7)
    # parts of at least 64 key tiles: 16K keys allow 2
    assert plan(1, 256, 16384, 20, 16128, 0, 0, 148) == (0, 20, 2)
    assert plan(1, 256, 8192, 20, 7936, 0, 0, 148) == (20, 0, 1)
    # more than half a wave left over: splitting it gains nothing
    assert plan(1, 256, 65536, 100, 65280, 0, 0, 148) == (100, 0, 1)
    # explicit parts: every item; parts past the last key tile are dropped
    assert plan(2, 300, 1000, 3, 700, 0, 5, 148) == (0, 12, 4)
    assert plan(1, 300, 1000, 3, 700, 0, 1, 148) == (6, 0, 1)
    # workspace: parts * split items * 256 rows * (D + 1) fp32
    ws = wp.prefill_split_workspace_size
    assert ws(1, 16384, 1048576, 28, 128, 1032192, 0, 0, 148) == 8 * 16 * 256 * 129 * 4
    assert ws(2, 300, 1000, 3, 64, 700, 0, 5, 148) == 4 * 12 * 256 * 65 * 4
    assert ws(1, 131072, 131072, 24, 128, 0, 0, 0, 148) == 0
    assert ws(1, 300, 1000, 3, 96, 700, 0, 5, 148) == 0
    w = wp.Window(64, 1e4, 1.0, 1)
    L = wp.lib()
    for S in (-1, 65):
        assert L.wpattn_prefill_split(ctypes.byref(w._c()), None, None, None, None, None, 1, 4, 4, 2,
                                      2, 0, 0, 0.0, S, None, 0, None) == wp.EINVAL
    with pytest.raises(wp.WpattnError):
        plan(1, 256, 1024, 2, 0, 0, 65, 148)


def test_decode_workspace_size_bounds_every_split_plan():
    w = wp.Window(128, 5e5, 1.0, 1)
    for B, Hq, Hkv, L in [(16, 24, 8, 131072), (1, 28, 4, 1048576), (3, 4, 2, 40), (1, 1, 1, 1)]:
        n = wp.decode_workspace_size(w, B, Hq, Hkv, L)
        assert n > 0 and n % 256 == 0
        assert n >= B * Hq * (128 + 2) * 4
