"""RoPE for inputs that arrive before their rotation, through the C ABI: the
rotation kernel against the oracle's exact rotation (each value within half a
bf16 ulp plus the float rotation error, and only a few values rounded the
other way from the oracle's bf16), decode with the rotation fused into the
query load (bitwise equal to rotate-then-decode, and against the oracle), and
prefill from pre-RoPE q and k (bitwise equal to rotate-then-prefill, and
against the oracle)."""
import math

import numpy as np
import pytest
import torch

import oracle
import rope_wavelength_sparsity_b200 as wp
from rope_wavelength_sparsity_b200 import inputs

from _parity import check_rows

pytestmark = pytest.mark.gpu

MAX_FLIP_FRACTION = 1e-3
# float rotation error allowed on top of the final rounding, relative to the
# pair's magnitude |x_p| + |x_{p+D/2}| (float cosines and products; large only
# where the two terms nearly cancel)
ROT_EPS = 4e-7


def _values(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def _compare_rotation(got_bits, x_bits, positions, base, what):
    """Every value within half a bf16 ulp of the exact rotation plus the float
    rotation error; at most a small fraction differing from the oracle's bf16."""
    want = oracle.rope(x_bits, positions, base=base)
    exact = oracle.rope(x_bits, positions, base=base, exact=True)
    got = _values(got_bits)
    x = _values(x_bits)
    P = x.shape[-1] // 2
    mag = np.abs(x[..., :P]) + np.abs(x[..., P:])
    mag = np.concatenate([mag, mag], axis=-1)
    ulp = np.abs(_values(want) - _values(np.asarray(want, dtype=np.uint32) + 1))
    bound = 0.5 * ulp + ROT_EPS * mag + 1e-30
    err = np.abs(got - exact)
    worst = float((err / bound).max())
    assert worst <= 1.0, f"{what}: error {worst:.2f}x the bound"
    frac = float((np.asarray(got_bits) != want).mean())
    assert frac <= MAX_FLIP_FRACTION, f"{what}: {frac:.2e} of the values differ from the oracle"
    return frac


@pytest.mark.parametrize("D,base,pos0", [(64, 1e4, 0), (128, 5e5, 0), (128, 1e7, 1032192),
                                         (64, 1e6, 123457)])
def test_rope_kernel_vs_oracle_contiguous(cuda_dev, D, base, pos0):
    B, N, H = 2, 300, 3
    x = inputs.randn_bf16((B, N, H, D), D + N)
    y = wp.rope(x.cuda(), base=base, pos0=pos0)
    torch.cuda.synchronize()
    xb = inputs.bits(x)
    for b in range(B):
        _compare_rotation(inputs.bits(y.cpu()[b]), xb[b], pos0 + np.arange(N), base,
                          f"D={D} base={base} b={b}")


@pytest.mark.parametrize("D", [64, 128])
def test_rope_kernel_explicit_positions_and_in_place(cuda_dev, D):
    B, N, H = 3, 200, 2
    x = inputs.randn_bf16((B, N, H, D), 7 * D)
    g = torch.Generator().manual_seed(D)
    pos = torch.randint(0, 2**31 - 1, (B, N), generator=g, dtype=torch.int64).to(torch.int32)
    pos[0, :5] = torch.tensor([0, 1, 2**31 - 2, 1048575, 131071], dtype=torch.int32)
    xd = x.cuda()
    y = wp.rope(xd, base=5e5, positions=pos.cuda())
    z = xd.clone()
    wp.rope(z, base=5e5, positions=pos.cuda(), out=z)      # in place
    torch.cuda.synchronize()
    assert torch.equal(y, z)
    xb = inputs.bits(x)
    for b in range(B):
        _compare_rotation(inputs.bits(y.cpu()[b]), xb[b], pos[b].numpy(), 5e5, f"D={D} b={b}")


QK_CASES = [
    # D, base, B, Nq, Nk, Hq, Hkv, q_pos0, k_pos0
    (64, 1e6, 2, 300, 300, 14, 2, 0, 0),        # head counts past and below the 4-head batch
    (128, 1e7, 1, 100, 700, 7, 1, 600, 0),      # chunked prefill: q at the end of k's range
    (128, 5e5, 3, 65, 33, 5, 3, 1032192, 77),
    (64, 1e4, 1, 129, 0, 4, 2, 5, 0),           # Nk = 0: q alone
]


@pytest.mark.parametrize("case", QK_CASES, ids=[str(i) for i in range(len(QK_CASES))])
def test_rope_qk_one_launch(cuda_dev, case):
    """The fused q and k rotation equals two separate rotations bit for bit, in
    place too, and each tensor is within the rotation bound of the oracle."""
    D, base, B, Nq, Nk, Hq, Hkv, q0, k0 = case
    s = len(str(case))
    q = inputs.randn_bf16((B, Nq, Hq, D), 50 * s + 1)
    k = inputs.randn_bf16((B, Nk, Hkv, D), 50 * s + 2)
    qd, kd = q.cuda(), k.cuda()
    qr, kr = wp.rope_qk(qd, kd, base=base, q_pos0=q0, k_pos0=k0)
    q1 = wp.rope(qd, base=base, pos0=q0)
    qi, ki = qd.clone(), kd.clone()
    wp.rope_qk(qi, ki, base=base, q_pos0=q0, k_pos0=k0, q_out=qi, k_out=ki)
    torch.cuda.synchronize()
    assert torch.equal(qr, q1) and torch.equal(qi, qr)
    if Nk > 0:
        k1 = wp.rope(kd, base=base, pos0=k0)
        torch.cuda.synchronize()
        assert torch.equal(kr, k1) and torch.equal(ki, kr)
    qb, kb = inputs.bits(q), inputs.bits(k)
    for b in range(B):
        _compare_rotation(inputs.bits(qr.cpu()[b]), qb[b], q0 + np.arange(Nq), base, f"q b={b}")
        if Nk > 0:
            _compare_rotation(inputs.bits(kr.cpu()[b]), kb[b], k0 + np.arange(Nk), base, f"k b={b}")


DEC_CASES = [
    # D, g, alpha, base, B, Hq, Hkv, L, kv_len
    (128, 1, 1.0, 5e5, 3, 24, 8, 1000, [1000, 1, 517]),
    (64, 8, 1.0, 1e6, 2, 14, 2, 3000, [3000, 2999]),
    (128, 8, 1.0, 1e7, 1, 28, 4, 5000, [5000]),
]


@pytest.mark.parametrize("case", DEC_CASES, ids=[str(i) for i in range(len(DEC_CASES))])
def test_decode_rope(cuda_dev, case):
    D, g, alpha, base, B, Hq, Hkv, L, kv_len = case
    seed = len(str(case)) + 300
    q = inputs.randn_bf16((B, Hq, D), seed * 10 + 1)
    kc = inputs.randn_bf16((B, L, Hkv, D), seed * 10 + 2)
    vc = inputs.randn_bf16((B, L, Hkv, D), seed * 10 + 3)
    win = wp.Window(D, base, alpha, g)
    qd, kd, vd = q.cuda(), kc.cuda(), vc.cuda()
    out, lse = wp.decode_rope(qd, kd, vd, kv_len, win)
    pos = torch.tensor([[n - 1] for n in kv_len], dtype=torch.int32).cuda()
    q_rot = wp.rope(qd.view(B, 1, Hq, D), base=base, positions=pos).view(B, Hq, D)
    out2, lse2 = wp.decode(q_rot, kd, vd, kv_len, win)
    assert wp.device_status() == wp.OK
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
    # the oracle on its own rotation of q
    qb = np.stack([oracle.rope(inputs.bits(q)[b:b + 1].reshape(1, Hq, D), [kv_len[b] - 1],
                               base=base)[0] for b in range(B)])
    rows = [(b, h) for b in range(B) for h in range(Hq)]
    o_ref, l_ref = oracle.decode_rows(qb, inputs.bits(kc), inputs.bits(vc), kv_len, Hq=Hq,
                                      Hkv=Hkv, base=base, alpha=alpha, g=g,
                                      scale=1.0 / math.sqrt(D), rows=rows)
    oc, lc = out.float().cpu(), lse.cpu()
    check_rows(np.stack([oc[b, h].numpy() for (b, h) in rows]),
               np.array([float(lc[b, h]) for (b, h) in rows]), o_ref, l_ref, str(case))


def test_decode_rope_with_positions(cuda_dev):
    D, B, Hq, Hkv, kv_len = 128, 2, 8, 2, [900, 300]
    L = max(kv_len)
    q = inputs.randn_bf16((B, Hq, D), 41).cuda()
    kc = inputs.randn_bf16((B, L, Hkv, D), 42).cuda()
    q_pos, k_pos = inputs.key_positions(kv_len, 5, "shuffled")
    win = wp.Window(D, 5e5, 1.0, 1)
    out, lse = wp.decode_rope(q, kc, kc, kv_len, win, q_pos=q_pos, k_pos=k_pos.cuda())
    pos = torch.tensor([[p] for p in q_pos], dtype=torch.int32).cuda()
    q_rot = wp.rope(q.view(B, 1, Hq, D), base=5e5, positions=pos).view(B, Hq, D)
    out2, lse2 = wp.decode_positions(q_rot, kc, kc, kv_len, q_pos, k_pos.cuda(), win)
    assert wp.device_status() == wp.OK
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


PRE_CASES = [
    # D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q_pos0, k_pos0
    (128, 1, 1.0, 5e5, 1, 3, 1, 300, 300, 0, 0),
    (64, 8, 1.0, 1e6, 2, 4, 2, 257, 257, 0, 0),
    (128, 8, 1.0, 1e7, 1, 2, 2, 100, 700, 600, 0),
    (64, 1, 2.0, 1e4, 1, 2, 1, 400, 400, 5000, 5000),
]


@pytest.mark.parametrize("case", PRE_CASES, ids=[str(i) for i in range(len(PRE_CASES))])
def test_prefill_rope(cuda_dev, case):
    D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q0, k0 = case
    s = len(str(case))
    q = inputs.randn_bf16((B, Nq, Hq, D), 100 * s + 1)
    k = inputs.randn_bf16((B, Nk, Hkv, D), 100 * s + 2)
    v = inputs.randn_bf16((B, Nk, Hkv, D), 100 * s + 3)
    win = wp.Window(D, base, alpha, g)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out, lse = wp.prefill_rope(qd, kd, vd, win, q_pos0=q0, k_pos0=k0)
    qr = wp.rope(qd, base=base, pos0=q0)
    kr = wp.rope(kd, base=base, pos0=k0)
    out2, lse2 = wp.prefill(qr, kr, vd, win, q_pos0=q0, k_pos0=k0)
    assert wp.device_status() == wp.OK
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
    qb = np.stack([oracle.rope(inputs.bits(q)[b], q0 + np.arange(Nq), base=base) for b in range(B)])
    kb = np.stack([oracle.rope(inputs.bits(k)[b], k0 + np.arange(Nk), base=base) for b in range(B)])
    rows = np.array([(b, h, t) for b in range(B) for h in range(Hq) for t in range(Nq)])
    o_ref, l_ref = oracle.attention_rows(qb, kb, inputs.bits(v), Hq=Hq, Hkv=Hkv, q_pos0=q0,
                                         k_pos0=k0, base=base, alpha=alpha, g=g,
                                         scale=1.0 / math.sqrt(D), rows=rows)
    bi, hi, ti = (torch.as_tensor(rows[:, i]) for i in range(3))
    check_rows(out.float().cpu()[bi, ti, hi].numpy(), lse.cpu()[bi, hi, ti].numpy(), o_ref, l_ref,
               str(case))


def test_rope_rejects_bad_args(cuda_dev):
    x = torch.zeros((1, 4, 1, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wp.WpattnError) as e:
        wp.rope(x, base=1e4)
    assert e.value.code == wp.EUNSUPPORTED
    with pytest.raises(wp.WpattnError) as e:
        wp.rope_qk(x, x, base=1e4)
    assert e.value.code == wp.EUNSUPPORTED
    y = torch.zeros((1, 4, 1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wp.WpattnError) as e:
        wp.rope_qk(y, y, base=1.0)
    assert e.value.code == wp.EINVAL
    with pytest.raises(wp.WpattnError) as e:
        wp.rope_qk(y, y, base=1e4, q_pos0=-1)
    assert e.value.code == wp.EINVAL
    q = torch.zeros((1, 256, 2, 64), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(wp.WpattnError) as e:
        wp.prefill_rope(q, q, q, wp.Window(64, 1e4, 1.0, 1), workspace=ws)
    assert e.value.code == wp.EWORKSPACE
