"""Guard regions around every buffer the kernels write or read (a bounds check
without compute-sanitizer).

Each output (out, lse, the decode workspace, the pair-major slabs, rotated
tensors) is carved out of a larger device buffer with 4 KB of seeded pattern
bytes before and after it, and is itself filled with NaN before the call.
Inputs sit inside NaN guards.  After each call, through the C ABI:
  * the guard bytes around every output are byte-identical to the pattern
    (no write ran past either end);
  * every output element was written and matches the oracle (a NaN left in an
    output, or a NaN read from an input guard, fails the comparison).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import rope_wavelength_sparsity_b200 as wp
from rope_wavelength_sparsity_b200 import inputs
from rope_wavelength_sparsity_b200 import distributed as wd

from _parity import check_rows

pytestmark = pytest.mark.gpu

GUARD = 4096            # bytes on each side of an output
IN_GUARD = 2048         # bf16 elements (4 KB) of NaN on each side of an input


class Guarded:
    """A device buffer: GUARD pattern bytes, the payload, GUARD pattern bytes."""

    def __init__(self, shape, dtype, seed):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        g = torch.Generator().manual_seed(seed)
        self.head = torch.randint(0, 256, (GUARD,), generator=g, dtype=torch.uint8)
        self.tail = torch.randint(0, 256, (GUARD,), generator=g, dtype=torch.uint8)
        self.buf = torch.empty(2 * GUARD + n, dtype=torch.uint8, device="cuda")
        self.buf[:GUARD] = self.head.cuda()
        self.buf[GUARD + n:] = self.tail.cuda()
        self.n = n
        self.t = self.buf[GUARD:GUARD + n].view(dtype).view(shape)
        self.t.fill_(float("nan") if dtype.is_floating_point else 0x5A)

    def check(self, what):
        torch.cuda.synchronize()
        assert torch.equal(self.buf[:GUARD].cpu(), self.head), f"{what}: write before the start"
        assert torch.equal(self.buf[GUARD + self.n:].cpu(), self.tail), f"{what}: write past the end"


def nan_guarded(x):
    """A copy of bf16 tensor x on the GPU with IN_GUARD NaN elements on each side."""
    n = x.numel()
    buf = torch.full((2 * IN_GUARD + n,), float("nan"), dtype=torch.bfloat16, device="cuda")
    t = buf[IN_GUARD:IN_GUARD + n].view(x.shape)
    t.copy_(x.cuda())
    return t


PREFILL_CASES = [
    # D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q_pos0
    (64, 1, 1.0, 1e4, 2, 4, 2, 300, 300, 0),
    (128, 8, 1.0, 1e7, 1, 6, 2, 200, 700, 500),
    (128, 1, 0.3, 10.0, 1, 3, 1, 130, 130, 0),
]


def _prefill_inputs(case, seed):
    D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q0 = case
    q = inputs.randn_bf16((B, Nq, Hq, D), seed + 1)
    k = inputs.randn_bf16((B, Nk, Hkv, D), seed + 2)
    v = inputs.randn_bf16((B, Nk, Hkv, D), seed + 3)
    return q, k, v


def _prefill_ref(q, k, v, case, rows=None):
    D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q0 = case
    if rows is None:
        rows = [(b, h, t) for b in range(B) for h in range(Hq) for t in range(Nq)]
    rows = np.asarray(rows, dtype=np.int64)
    o, l = oracle.attention_rows(inputs.bits(q), inputs.bits(k), inputs.bits(v), Hq=Hq, Hkv=Hkv,
                                 q_pos0=q0, base=base, alpha=alpha, g=g, scale=1 / math.sqrt(D),
                                 rows=rows)
    return rows, o, l


def _compare_prefill(out, lse, rows, o_ref, l_ref, what):
    bi, hi, ti = (torch.as_tensor(rows[:, i]) for i in range(3))
    check_rows(out.float().cpu()[bi, ti, hi].numpy(), lse.cpu()[bi, hi, ti].numpy(), o_ref, l_ref,
               what)


@pytest.mark.parametrize("case", PREFILL_CASES, ids=[str(i) for i in range(len(PREFILL_CASES))])
def test_prefill_guards(cuda_dev, case):
    D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q0 = case
    q, k, v = _prefill_inputs(case, 7000 + len(str(case)))
    win = wp.Window(D, base, alpha, g)
    out = Guarded((B, Nq, Hq, D), torch.bfloat16, 1)
    lse = Guarded((B, Hq, Nq), torch.float32, 2)
    wp.prefill(nan_guarded(q), nan_guarded(k), nan_guarded(v), win, q_pos0=q0, out=out.t,
               lse=lse.t, check=True)
    out.check("prefill out")
    lse.check("prefill lse")
    rows, o_ref, l_ref = _prefill_ref(q, k, v, case)
    _compare_prefill(out.t, lse.t, rows, o_ref, l_ref, f"prefill {case}")


def test_prefill_masked_and_positions_guards(cuda_dev):
    case = PREFILL_CASES[0]
    D, g, alpha, base, B, Hq, Hkv, Nq, Nk, q0 = case
    q, k, v = _prefill_inputs(case, 7100)
    qg, kg, vg = nan_guarded(q), nan_guarded(k), nan_guarded(v)
    win = wp.Window(D, base, alpha, g)
    # an all-ones mask: the same result as the plain call
    nqb, nkb = -(-Nq // 128), -(-Nk // 128)
    mask = torch.ones((B, Hq, nqb, nkb), dtype=torch.bool, device="cuda")
    out = Guarded((B, Nq, Hq, D), torch.bfloat16, 3)
    lse = Guarded((B, Hq, Nq), torch.float32, 4)
    wp.prefill_masked(qg, kg, vg, mask, win, out=out.t, lse=lse.t)
    assert wp.device_status() == wp.OK
    out.check("masked out")
    lse.check("masked lse")
    rows, o_ref, l_ref = _prefill_ref(q, k, v, case)
    _compare_prefill(out.t, lse.t, rows, o_ref, l_ref, "masked")
    # the workload's own contiguous positions through the explicit-positions kernel
    qp = torch.arange(Nq, dtype=torch.int32, device="cuda").repeat(B, 1)
    kp = torch.arange(Nk, dtype=torch.int32, device="cuda").repeat(B, 1)
    out2 = Guarded((B, Nq, Hq, D), torch.bfloat16, 5)
    lse2 = Guarded((B, Hq, Nq), torch.float32, 6)
    wp.prefill_positions(qg, kg, vg, qp, kp, win, out=out2.t, lse=lse2.t)
    assert wp.device_status() == wp.OK
    out2.check("positions out")
    lse2.check("positions lse")
    _compare_prefill(out2.t, lse2.t, rows, o_ref, l_ref, "positions")


DECODE_CASES = [
    # D, g, alpha, base, B, Hq, Hkv, L, kv_len
    (128, 1, 1.0, 5e5, 3, 6, 2, 1000, [1000, 1, 517]),
    (64, 8, 1.0, 1e6, 2, 14, 2, 700, [64, 700]),
]


def _decode_ref(q, kc, vc, kv_len, case):
    D, g, alpha, base, B, Hq, Hkv, L, _ = case
    rows = [(b, h) for b in range(B) for h in range(Hq)]
    o, l = oracle.decode_rows(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len, Hq=Hq,
                              Hkv=Hkv, base=base, alpha=alpha, g=g, scale=1 / math.sqrt(D),
                              rows=rows)
    return rows, o, l


def _compare_decode(out, lse, rows, o_ref, l_ref, what):
    oc, lc = out.float().cpu(), lse.cpu()
    check_rows(np.stack([oc[b, h].numpy() for (b, h) in rows]),
               np.array([float(lc[b, h]) for (b, h) in rows]), o_ref, l_ref, what)


@pytest.mark.parametrize("case", DECODE_CASES, ids=[str(i) for i in range(len(DECODE_CASES))])
def test_decode_layouts_guards(cuda_dev, case):
    D, g, alpha, base, B, Hq, Hkv, L, kv_len = case
    seed = 7200 + len(str(case))
    q = inputs.randn_bf16((B, Hq, D), seed + 1)
    kc = inputs.randn_bf16((B, L, Hkv, D), seed + 2)
    vc = inputs.randn_bf16((B, L, Hkv, D), seed + 3)
    qg, kg, vg = nan_guarded(q), nan_guarded(kc), nan_guarded(vc)
    win = wp.Window(D, base, alpha, g)
    rows, o_ref, l_ref = _decode_ref(q, kc, vc, kv_len, case)
    nws = wp.decode_workspace_size(win, B, Hq, Hkv, L)
    # contiguous cache
    out = Guarded((B, Hq, D), torch.bfloat16, 11)
    lse = Guarded((B, Hq), torch.float32, 12)
    ws = Guarded((nws,), torch.uint8, 13)
    wp.decode(qg, kg, vg, kv_len, win, out=out.t, lse=lse.t, workspace=ws.t, check=True)
    for x, name in ((out, "out"), (lse, "lse"), (ws, "workspace")):
        x.check(f"decode {name}")
    _compare_decode(out.t, lse.t, rows, o_ref, l_ref, f"decode {case}")
    # pair-major K: the conversion's output and the decode's outputs
    slabs = Guarded((B, Hkv, D // 16, L, 16), torch.bfloat16, 14)
    wp.kcache_to_pairmajor(kg, out=slabs.t)
    slabs.check("pair-major slabs")
    out = Guarded((B, Hq, D), torch.bfloat16, 15)
    lse = Guarded((B, Hq), torch.float32, 16)
    ws = Guarded((nws,), torch.uint8, 17)
    wp.decode_pairmajor(qg, slabs.t, vg, kv_len, win, out=out.t, lse=lse.t, workspace=ws.t)
    assert wp.device_status() == wp.OK
    for x, name in ((out, "out"), (lse, "lse"), (ws, "workspace")):
        x.check(f"pair-major decode {name}")
    _compare_decode(out.t, lse.t, rows, o_ref, l_ref, f"pair-major {case}")
    # paged cache (16-row pages, shuffled; unused pool rows are NaN)
    page = 16
    table, num_pages = inputs.page_layout(kv_len, page, seed=seed)
    kp = inputs.scatter_to_pages(kg, kv_len, table, page, num_pages)
    vp = inputs.scatter_to_pages(vg, kv_len, table, page, num_pages)
    nws_pg = wp.decode_workspace_size(win, B, Hq, Hkv, table.shape[1] * page)
    out = Guarded((B, Hq, D), torch.bfloat16, 18)
    lse = Guarded((B, Hq), torch.float32, 19)
    ws = Guarded((nws_pg,), torch.uint8, 20)
    wp.decode_paged(qg, kp, vp, table.cuda(), kv_len, win, out=out.t, lse=lse.t, workspace=ws.t)
    assert wp.device_status() == wp.OK
    for x, name in ((out, "out"), (lse, "lse"), (ws, "workspace")):
        x.check(f"paged decode {name}")
    _compare_decode(out.t, lse.t, rows, o_ref, l_ref, f"paged {case}")


def test_shards_merge_and_rope_guards(cuda_dev):
    D, g, alpha, base, B, Hq, Hkv, shard, world = 128, 1, 1.0, 5e5, 2, 6, 2, 300, 3
    kv_len = [900, 450]
    L = shard * world
    q = inputs.randn_bf16((B, Hq, D), 7301)
    kc = inputs.randn_bf16((B, L, Hkv, D), 7302)
    vc = inputs.randn_bf16((B, L, Hkv, D), 7303)
    win = wp.Window(D, base, alpha, g)
    qg = nan_guarded(q)
    parts_o = Guarded((world, B, Hq, D), torch.bfloat16, 21)
    parts_l = Guarded((world, B, Hq), torch.float32, 22)
    for r in range(world):
        k_pos0, n = wd.shard_keys(kv_len, r, shard)
        ks = nan_guarded(kc[:, r * shard:(r + 1) * shard].contiguous())
        vs = nan_guarded(vc[:, r * shard:(r + 1) * shard].contiguous())
        wp.decode_shard(qg, ks, vs, n, [x - 1 for x in kv_len], k_pos0, win,
                        out=parts_o.t[r], lse=parts_l.t[r])
    out = Guarded((B, Hq, D), torch.bfloat16, 23)
    lse = Guarded((B, Hq), torch.float32, 24)
    wp.merge_lse(parts_o.t, parts_l.t, out=out.t, lse=lse.t)
    assert wp.device_status() == wp.OK
    for x, name in ((parts_o, "shard outs"), (parts_l, "shard lses"), (out, "merged out"),
                    (lse, "merged lse")):
        x.check(name)
    rows = [(b, h) for b in range(B) for h in range(Hq)]
    o_ref, l_ref = oracle.decode_rows(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len,
                                      Hq=Hq, Hkv=Hkv, base=base, alpha=alpha, g=g,
                                      scale=1 / math.sqrt(D), rows=rows)
    _compare_decode(out.t, lse.t, rows, o_ref, l_ref, "shards merged")
    # the rotation kernel: its guarded output bit for bit equal to a plain call's (its
    # values against the oracle are the rotation tests' business)
    x = inputs.randn_bf16((2, 77, 3, 64), 7304)
    rot = Guarded((2, 77, 3, 64), torch.bfloat16, 25)
    wp.rope(nan_guarded(x), base=1e4, pos0=5, out=rot.t)
    rot.check("rope out")
    plain = wp.rope(x.cuda(), base=1e4, pos0=5)
    assert torch.equal(rot.t.view(torch.int16), plain.view(torch.int16))
