"""Decode parity on the GPU: split-KV kernel + combine (through the C ABI)
vs the oracle, every (sequence, head), with ragged cache lengths, GQA group
sizes 1..16, both granularities and the method's degenerate windows."""
import pytest
import torch

import rope_wavelength_sparsity_b200 as wp
from rope_wavelength_sparsity_b200 import inputs

from _parity import decode_parity

pytestmark = pytest.mark.gpu

CASES = [
    # D, g, alpha, base, B, Hq, Hkv, L, kv_len
    (128, 1, 1.0, 5e5, 3, 24, 8, 1000, [1000, 1, 517]),
    (64, 8, 1.0, 1e6, 2, 14, 2, 3000, [3000, 2999]),
    (128, 8, 1.0, 1e7, 1, 28, 4, 5000, [5000]),
    (128, 1, float("inf"), 5e5, 2, 16, 1, 700, [700, 64]),     # GQA 16: two head chunks
    (64, 1, 1e-3, 1e4, 2, 4, 4, 900, [900, 33]),                # everything pruned far away
    (128, 1, 1.0, 10.0, 2, 6, 2, 1500, [1500, 777]),            # many partial chunks
    (64, 1, 2.0, 1e4, 4, 9, 3, 2048, [2048, 1, 2, 1999]),       # GQA 3, tiny lengths
    (128, 8, 0.05, 1e4, 1, 12, 1, 4100, [4100]),                # GQA 12: chunks of 6
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_decode_cases_all_rows(cuda_dev, case):
    D, g, alpha, base, B, Hq, Hkv, L, kv_len = case
    seed = len(str(case))
    q = inputs.randn_bf16((B, Hq, D), seed * 10 + 1)
    kc = inputs.randn_bf16((B, L, Hkv, D), seed * 10 + 2)
    vc = inputs.randn_bf16((B, L, Hkv, D), seed * 10 + 3)
    decode_parity(q, kc, vc, kv_len, Hq=Hq, Hkv=Hkv, D=D, base=base, alpha=alpha, g=g,
                  what=str(case))


def test_decode_equals_last_row_of_prefill(cuda_dev):
    """A decode step at kv_len = N is the last row of a prefill over N keys."""
    D, Hq, Hkv, N = 128, 8, 2, 777
    q = inputs.randn_bf16((1, N, Hq, D), 71)
    k = inputs.randn_bf16((1, N, Hkv, D), 72)
    v = inputs.randn_bf16((1, N, Hkv, D), 73)
    win = wp.Window(D, 5e5, 1.0, 1)
    out_p, lse_p = wp.prefill(q.cuda(), k.cuda(), v.cuda(), win)
    out_d, lse_d = wp.decode(q[:, -1].contiguous().cuda(), k.cuda(), v.cuda(), [N], win)
    torch.cuda.synchronize()
    assert (out_p[0, -1].float() - out_d[0].float()).abs().max().item() <= 1e-2
    assert (lse_p[0, :, -1] - lse_d[0]).abs().max().item() <= 2e-3


def test_decode_workspace_too_small(cuda_dev):
    D, B, Hq, Hkv, L = 64, 1, 2, 1, 100
    win = wp.Window(D, 1e4, 1.0, 1)
    q = inputs.randn_bf16((B, Hq, D), 1).cuda()
    kc = inputs.randn_bf16((B, L, Hkv, D), 2).cuda()
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(wp.WpattnError) as e:
        wp.decode(q, kc, kc, [L], win, workspace=ws)
    assert e.value.code == wp.EWORKSPACE


def test_decode_maximum_batch(cuda_dev):
    """The largest batch one call takes (1024 sequences), with lengths from 1 to 64:
    every row against the oracle; one more sequence is refused."""
    import numpy as np
    import oracle
    from _parity import check_rows
    B, Hq, Hkv, D, L = 1024, 4, 2, 64, 64
    q = inputs.randn_bf16((B, Hq, D), 81)
    kc = inputs.randn_bf16((B, L, Hkv, D), 82)
    vc = inputs.randn_bf16((B, L, Hkv, D), 83)
    kv_len = [1 + (7 * b) % L for b in range(B)]
    win = wp.Window(D, 1e4, 1.0, 1)
    out, lse = wp.decode(q.cuda(), kc.cuda(), vc.cuda(), kv_len, win)
    assert wp.device_status() == wp.OK
    o_ref, l_ref = oracle.decode_rows(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len,
                                      Hq=Hq, Hkv=Hkv, base=1e4, alpha=1.0, g=1,
                                      scale=1.0 / D ** 0.5)
    check_rows(out.float().cpu().reshape(B * Hq, D).numpy(), lse.cpu().reshape(-1).numpy(),
               o_ref, l_ref, "B=1024")
    q1 = torch.zeros((B + 1, Hq, D), dtype=torch.bfloat16, device="cuda")
    k1 = torch.zeros((B + 1, 8, Hkv, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wp.WpattnError) as e:
        wp.decode(q1, k1, k1, [8] * (B + 1), win)
    assert e.value.code == wp.EUNSUPPORTED
