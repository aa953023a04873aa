"""Prefill with explicit per-token positions, through the C ABI: contiguous
positions give the plain prefill bit for bit; positions with gaps, repeated
positions and chunked-prefill layouts against the oracle on every row; keys
all after the queries give empty rows."""
import math

import numpy as np
import pytest
import torch

import oracle
import rope_wavelength_sparsity_b200 as wp
from rope_wavelength_sparsity_b200 import inputs

from _parity import check_rows

pytestmark = pytest.mark.gpu


def _qkv(B, Nq, Nk, Hq, Hkv, D, seed):
    return (inputs.randn_bf16((B, Nq, Hq, D), 100 * seed + 1),
            inputs.randn_bf16((B, Nk, Hkv, D), 100 * seed + 2),
            inputs.randn_bf16((B, Nk, Hkv, D), 100 * seed + 3))


def _run_and_check(q, k, v, qp, kp, *, D, g, alpha, base, Hq, Hkv, what, rows=None):
    B, Nq = q.shape[0], q.shape[1]
    win = wp.Window(D, base, alpha, g)
    out, lse = wp.prefill_positions(q.cuda(), k.cuda(), v.cuda(), qp.cuda(), kp.cuda(), win)
    assert wp.device_status() == wp.OK
    if rows is None:
        rows = [(b, h, t) for b in range(B) for h in range(Hq) for t in range(Nq)]
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    o_ref, l_ref = oracle.attention_positions(inputs.bits(q), inputs.bits(k), inputs.bits(v),
                                              qp.numpy(), kp.numpy(), Hq=Hq, Hkv=Hkv, base=base,
                                              alpha=alpha, g=g, scale=1.0 / math.sqrt(D), rows=rows)
    bi, hi, ti = (torch.as_tensor(rows[:, i]) for i in range(3))
    return check_rows(out.float().cpu()[bi, ti, hi].numpy(), lse.cpu()[bi, hi, ti].numpy(),
                      o_ref, l_ref, what)


@pytest.mark.parametrize("D,g,Nq,Nk,q0,k0", [(64, 8, 520, 520, 0, 0), (128, 1, 300, 700, 400, 0),
                                             (128, 8, 257, 1000, 5000, 4257), (64, 1, 129, 129, 0, 0)])
def test_contiguous_positions_equal_prefill(cuda_dev, D, g, Nq, Nk, q0, k0):
    B, Hq, Hkv = 2, 4, 2
    q, k, v = _qkv(B, Nq, Nk, Hq, Hkv, D, seed=D + Nq)
    win = wp.Window(D, 1e4, 1.0, g)
    qp = (q0 + torch.arange(Nq, dtype=torch.int32)).repeat(B, 1)
    kp = (k0 + torch.arange(Nk, dtype=torch.int32)).repeat(B, 1)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    a = wp.prefill_positions(qd, kd, vd, qp.cuda(), kp.cuda(), win)
    b = wp.prefill(qd, kd, vd, win, q_pos0=q0, k_pos0=k0)
    assert wp.device_status() == wp.OK
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


CASES = [
    # D, g, alpha, base, B, Hq, Hkv, Nq, Nk, layout
    (128, 1, 1.0, 5e5, 1, 3, 1, 600, 600, "gaps"),
    (64, 8, 1.0, 1e6, 2, 4, 2, 520, 520, "gaps"),
    (128, 8, 1.0, 1e7, 1, 2, 2, 300, 1500, "chunk"),
    (64, 1, 2.0, 1e4, 1, 2, 1, 700, 700, "repeats"),
    (128, 1, 0.3, 1e4, 1, 2, 1, 650, 650, "gaps"),
    (64, 1, 1.0, 10.0, 1, 2, 2, 333, 333, "repeats"),
    (128, 1, 1.0, 5e5, 2, 2, 1, 400, 400, "wide"),
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_positions_vs_oracle(cuda_dev, case):
    D, g, alpha, base, B, Hq, Hkv, Nq, Nk, layout = case
    seed = len(str(case))
    q, k, v = _qkv(B, Nq, Nk, Hq, Hkv, D, seed=seed)
    if layout == "chunk":
        # the queries are the last Nq of the keys (a chunk appended to a cache with gaps)
        kp = inputs.sorted_positions(B, Nk, seed, span=2.5)
        qp = kp[:, Nk - Nq:].contiguous()
    elif layout == "repeats":
        kp = inputs.sorted_positions(B, Nk, seed, span=1.5, repeats=True)
        qp = kp[:, :Nq].contiguous()
    elif layout == "wide":
        # gaps of up to 2 * 10^6 positions: most tiles span many wavelengths
        gen = torch.Generator().manual_seed(seed)
        gaps = torch.randint(1, 2_000_000, (B, Nk), generator=gen)
        kp = torch.cumsum(gaps, 1).to(torch.int32)
        qp = kp[:, :Nq].contiguous()
    else:
        kp = inputs.sorted_positions(B, Nk, seed, span=3.0)
        qp = kp[:, :Nq].contiguous()
    _run_and_check(q, k, v, qp, kp, D=D, g=g, alpha=alpha, base=base, Hq=Hq, Hkv=Hkv,
                   what=str(case))


def test_positions_queries_before_all_keys(cuda_dev):
    D, B, Hq, Hkv, Nq, Nk = 64, 1, 2, 1, 600, 300
    q, k, v = _qkv(B, Nq, Nk, Hq, Hkv, D, seed=77)
    qp = torch.arange(Nq, dtype=torch.int32)[None] * 2              # 0 .. 1198
    kp = 700 + torch.arange(Nk, dtype=torch.int32)[None]             # 700 .. 999
    _run_and_check(q, k, v, qp, kp, D=D, g=1, alpha=1.0, base=1e4, Hq=Hq, Hkv=Hkv,
                   what="late keys")


def test_positions_full_size_sampled(cuda_dev):
    """Llama-3.2-3B-shaped 32K prefill whose keys keep every other position (16K keys
    over 32K positions), queries the last 4K of them; sampled rows."""
    D, g, B, Hq, Hkv, Nk, Nq = 128, 1, 1, 4, 1, 16384, 4096
    q, k, v = _qkv(B, Nq, Nk, Hq, Hkv, D, seed=91)
    kp = inputs.sorted_positions(B, Nk, 91, span=2.0)
    qp = kp[:, Nk - Nq:].contiguous()
    rng = np.random.default_rng(5)
    rows = [(0, int(rng.integers(0, Hq)), int(t)) for t in
            np.concatenate([[0, 127, 128, Nq - 1], rng.integers(0, Nq, 40)])]
    _run_and_check(q, k, v, qp, kp, D=D, g=g, alpha=1.0, base=5e5, Hq=Hq, Hkv=Hkv,
                   what="32K gaps", rows=rows)


def test_positions_reject_bad_strides(cuda_dev):
    D = 64
    q = inputs.randn_bf16((1, 64, 1, D), 1).cuda()
    qp = torch.zeros((1, 32), dtype=torch.int32, device="cuda")      # shorter than Nq
    kp = torch.zeros((1, 128), dtype=torch.int32, device="cuda")
    with pytest.raises(wp.WpattnError) as e:
        wp.prefill_positions(q, q, q, qp, kp, wp.Window(D, 1e4, 1.0, 1))
    assert e.value.code == wp.EINVAL
