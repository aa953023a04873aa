"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module holds no part of the method's arithmetic: it only draws random
tensors with the shapes and value distributions of the workloads.  The
planted-key fixture scales one key so that its *longest-wavelength* pairs
line up with a chosen query; which pairs those are is a fixed structural
choice (the last ``PLANT_PAIRS`` pair indices), not a window computation.

All tensors are bf16 in the layouts the library takes:
  prefill  q [B, Nq, Hq, D], k/v [B, Nk, Hkv, D]
  decode   q [B, Hq, D],     k/v cache [B, L, Hkv, D]
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

PLANT_PAIRS = 8  # pair indices P-8 .. P-1: the 8 longest RoPE wavelengths


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, RoPE window parameters and input recipe."""
    name: str
    kind: str                      # "prefill" or "decode"
    B: int
    Hq: int
    Hkv: int
    D: int
    Nq: int                        # prefill queries (decode: 1)
    Nk: int                        # prefill keys / decode cache length
    base: float
    alpha: float
    g: int
    q_pos0: int = 0
    k_pos0: int = 0
    pair_lognormal_sigma: float = 0.0   # >0: per-(head, pair) magnitudes for q and k
    plant_key: bool = False
    extra: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


# Workloads of the pages' evaluation models, as single-layer attention shapes.
WORKLOADS = {
    "tiny": Workload("tiny", "prefill", 1, 1, 1, 64, 256, 256, 1e4, 1.0, 1),
    "qwen2.5-0.5b-32k": Workload("qwen2.5-0.5b-32k", "prefill", 1, 14, 2, 64, 32768, 32768,
                                 1e6, 1.0, 8, pair_lognormal_sigma=0.5),
    "llama3.2-3b-128k-a1": Workload("llama3.2-3b-128k-a1", "prefill", 1, 24, 8, 128, 131072,
                                    131072, 5e5, 1.0, 1, plant_key=True),
    "llama3.2-3b-128k-a2": Workload("llama3.2-3b-128k-a2", "prefill", 1, 24, 8, 128, 131072,
                                    131072, 5e5, 2.0, 1, plant_key=True),
    "llama3.2-3b-decode-128k": Workload("llama3.2-3b-decode-128k", "decode", 16, 24, 8, 128, 1,
                                        131072, 5e5, 1.0, 1),
    "qwen2.5-7b-1m-prefill": Workload("qwen2.5-7b-1m-prefill", "prefill", 1, 28, 4, 128, 16384,
                                      1048576, 1e7, 1.0, 8, q_pos0=1048576 - 16384),
    "qwen2.5-7b-1m-decode": Workload("qwen2.5-7b-1m-decode", "decode", 1, 28, 4, 128, 1,
                                     1048576, 1e7, 1.0, 8),
    # reduced shapes of the same kernels, for profiler captures (inputs still larger than L2)
    "llama3.2-3b-32k-a1": Workload("llama3.2-3b-32k-a1", "prefill", 1, 24, 8, 128, 32768, 32768,
                                   5e5, 1.0, 1),
    "llama3.2-3b-decode-32k": Workload("llama3.2-3b-decode-32k", "decode", 4, 24, 8, 128, 1,
                                       32768, 5e5, 1.0, 1),
    "qwen2.5-7b-64k-chunk": Workload("qwen2.5-7b-64k-chunk", "prefill", 1, 28, 4, 128, 16384,
                                     65536, 1e7, 1.0, 8, q_pos0=65536 - 16384),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn_bf16(shape, seed: int, device="cpu") -> torch.Tensor:
    """i.i.d. N(0, 1) rounded to bf16."""
    x = torch.randn(shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return x.to(torch.bfloat16)


def _pair_magnitudes(H: int, D: int, sigma: float, seed: int, device) -> torch.Tensor:
    """[H, D] multipliers: one LogNormal(0, sigma) draw per (head, pair), shared by dims p, p+D/2."""
    m = torch.exp(sigma * torch.randn((H, D // 2), generator=_gen(seed, device),
                                      device=device, dtype=torch.float32))
    return torch.cat([m, m], dim=1)


def prefill_inputs(w: Workload, seed: int = 0, device="cpu"):
    """(q, k, v, planted) for a prefill workload.

    Generator seeds are 16*seed + {1: q, 2: k, 3: v, 4/5: q/k pair magnitudes, 6: planted key}.
    """
    s = seed * 16
    shape_q = (w.B, w.Nq, w.Hq, w.D)
    shape_k = (w.B, w.Nk, w.Hkv, w.D)
    if w.pair_lognormal_sigma > 0:
        q = torch.randn(shape_q, generator=_gen(s + 1, device), device=device)
        k = torch.randn(shape_k, generator=_gen(s + 2, device), device=device)
        q *= _pair_magnitudes(w.Hq, w.D, w.pair_lognormal_sigma, s + 4, device)
        k *= _pair_magnitudes(w.Hkv, w.D, w.pair_lognormal_sigma, s + 5, device)
        q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
    else:
        q = randn_bf16(shape_q, s + 1, device)
        k = randn_bf16(shape_k, s + 2, device)
    v = randn_bf16(shape_k, s + 3, device)
    planted = []
    if w.plant_key:
        planted = plant_keys(q, k, Hq=w.Hq, Hkv=w.Hkv, scale=w.scale, seed=s + 6)
    return q, k, v, planted


def plant_keys(q: torch.Tensor, k: torch.Tensor, *, Hq: int, Hkv: int, scale: float, seed: int):
    """Plant one aligned key per kv head (in place); returns [(b, hq, t, kvh, j*)].

    For kv head kvh the probe query is the last row (t = Nq-1) of the group's
    first query head.  A key index j* ~ U[0, Nk/2) is drawn; its last
    ``PLANT_PAIRS`` pairs are set to c * (the query's same pairs), with c chosen
    so that those pairs alone add ln(Nk) + 10 to the scaled score.  The other
    pairs of the key stay random.  Values are rounded to bf16 afterwards.
    """
    B, Nq, _, D = q.shape
    Nk = k.shape[1]
    P = D // 2
    G = Hq // Hkv
    gen = _gen(seed, "cpu")
    lo = list(range(P - PLANT_PAIRS, P)) + list(range(D - PLANT_PAIRS, D))
    idx = torch.tensor(lo, device=q.device)
    planted = []
    for b in range(B):
        for kvh in range(Hkv):
            hq = kvh * G
            t = Nq - 1
            j = int(torch.randint(0, max(1, Nk // 2), (1,), generator=gen).item())
            qv = q[b, t, hq].float()
            qsel = qv[idx]
            target = math.log(Nk) + 10.0
            c = target / (scale * float((qsel * qsel).sum()))
            row = k[b, j, kvh].float()
            row[idx] = c * qsel
            k[b, j, kvh] = row.to(torch.bfloat16)
            planted.append((b, hq, t, kvh, j))
    return planted


def decode_inputs(w: Workload, seed: int = 0, device="cpu"):
    """(q [B,Hq,D], k_cache, v_cache [B,L,Hkv,D], kv_len [B]) for a decode workload.

    Every sequence is full (kv_len = L) unless ``w.extra['ragged']`` asks for
    lengths drawn uniformly from [1, L].
    """
    s = seed * 16
    q = randn_bf16((w.B, w.Hq, w.D), s + 7, device)
    kc = randn_bf16((w.B, w.Nk, w.Hkv, w.D), s + 8, device)
    vc = randn_bf16((w.B, w.Nk, w.Hkv, w.D), s + 9, device)
    if w.extra.get("ragged"):
        kv_len = torch.randint(1, w.Nk + 1, (w.B,), generator=_gen(s + 10, "cpu"),
                               dtype=torch.int32)
    else:
        kv_len = torch.full((w.B,), w.Nk, dtype=torch.int32)
    return q, kc, vc, kv_len


def bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (CPU), the form the oracle reads."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


def page_layout(kv_len, page_size: int, seed: int, spare_pages: int = 3):
    """(block_table int32 [B, max_pages], num_pages) of a shuffled page pool.

    Sequence b gets ceil(kv_len[b] / page_size) distinct pages drawn in random
    order from a pool with ``spare_pages`` pages nobody uses; entries past a
    sequence's last page are -1 (a reader that touched them would be caught).
    """
    kv = [int(x) for x in kv_len]
    need = [(n + page_size - 1) // page_size for n in kv]
    max_pages = max(need)
    num_pages = sum(need) + spare_pages
    perm = torch.randperm(num_pages, generator=_gen(seed, "cpu")).to(torch.int32)
    table = torch.full((len(kv), max_pages), -1, dtype=torch.int32)
    at = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[at:at + n]
        at += n
    return table, num_pages


def _page_rows(n: int, table_row: torch.Tensor, page_size: int, device) -> torch.Tensor:
    """Pool row (page * page_size + row in page) of cache rows 0..n-1 of one sequence."""
    j = torch.arange(n, device=device)
    return table_row.to(device).long()[j // page_size] * page_size + j % page_size


def scatter_to_pages(cache: torch.Tensor, kv_len, block_table: torch.Tensor, page_size: int,
                     num_pages: int) -> torch.Tensor:
    """[B, L, Hkv, D] cache -> pool [num_pages, page_size, Hkv, D] on the cache's
    device: rows j < kv_len[b] go to their page; every other row of the pool
    (unused pages, the tail of a sequence's last page) is NaN, so a kernel that
    read one would show it."""
    B, L, Hkv, D = cache.shape
    pool = torch.full((num_pages * page_size, Hkv, D), float("nan"), dtype=cache.dtype,
                      device=cache.device)
    for b in range(B):
        n = int(kv_len[b])
        pool[_page_rows(n, block_table[b], page_size, cache.device)] = cache[b, :n]
    return pool.view(num_pages, page_size, Hkv, D)


def gather_pages(pool: torch.Tensor, kv_len, block_table: torch.Tensor) -> torch.Tensor:
    """The [B, max_pages * page_size, Hkv, D] cache a block table describes, on the
    pool's device (rows past a sequence's last page are NaN)."""
    num_pages, page_size, Hkv, D = pool.shape
    B, max_pages = block_table.shape
    out = torch.full((B, max_pages * page_size, Hkv, D), float("nan"), dtype=pool.dtype,
                     device=pool.device)
    flat = pool.reshape(num_pages * page_size, Hkv, D)
    for b in range(B):
        n = (int(kv_len[b]) + page_size - 1) // page_size * page_size
        out[b, :n] = flat[_page_rows(n, block_table[b], page_size, pool.device)]
    return out


def key_positions(kv_len, seed: int, mode: str = "evicted", span: float = 4.0):
    """(q_pos [B] ints, k_pos int32 [B, max kv_len]) for caches that dropped tokens.

    ``evicted``: each sequence keeps kv_len[b] of the first round(span * kv_len[b])
    positions (a random subset, sorted); the query comes right after the last
    kept key, so the most recent key is always kept.  ``shuffled``: the same
    positions in random cache order.  ``future``: as ``shuffled`` but about a
    tenth of the keys sit after the query (they must be left out).
    Unused columns are -1 (never read).
    """
    g = _gen(seed, "cpu")
    kv = [int(x) for x in kv_len]
    k_pos = torch.full((len(kv), max(kv)), -1, dtype=torch.int32)
    q_pos = []
    for b, n in enumerate(kv):
        total = max(n, int(round(span * n)))
        keep = torch.randperm(total, generator=g)[:n].sort().values.to(torch.int32)
        qp = int(keep[-1]) + 1
        if mode in ("shuffled", "future"):
            keep = keep[torch.randperm(n, generator=g)]
        if mode == "future":
            late = torch.rand(n, generator=g) < 0.1
            keep = torch.where(late, qp + 1 + torch.randint(0, 1000, (n,), generator=g,
                                                            dtype=torch.int32), keep)
        k_pos[b, :n] = keep
        q_pos.append(qp)
    return q_pos, k_pos


def vertical_slash_mask(B: int, Hq: int, Nq: int, Nk: int, seed: int, q_pos0: int = 0,
                        k_pos0: int = 0, n_vertical: int = 4, band: int = 16, block: int = 128):
    """bool [B, Hq, ceil(Nq/block), ceil(Nk/block)] block mask of the MInference
    'vertical-slash' shape: per head, key tile 0 (the sink) and n_vertical - 1
    other key tiles drawn at random, attended by every query tile, plus a band
    of ``band`` key tiles ending at each query tile's diagonal tile."""
    g = _gen(seed, "cpu")
    nqb, nkb = -(-Nq // block), -(-Nk // block)
    m = torch.zeros((B, Hq, nqb, nkb), dtype=torch.bool)
    for b in range(B):
        for h in range(Hq):
            cols = [0] + torch.randint(0, nkb, (max(0, n_vertical - 1),), generator=g).tolist()
            m[b, h, :, cols] = True
            for qb in range(nqb):
                diag = (q_pos0 - k_pos0 + qb * block + block - 1) // block
                lo, hi = max(0, diag - band + 1), min(nkb - 1, diag)
                if hi >= lo:
                    m[b, h, qb, lo:hi + 1] = True
    return m


def sorted_positions(B: int, N: int, seed: int, span: float = 3.0, repeats: bool = False):
    """int32 [B, N] non-decreasing positions: each row keeps N of the first
    round(span * N) positions (a random sorted subset: a sequence with dropped
    tokens).  ``repeats`` draws with replacement instead, so equal positions
    occur (tokens sharing a position)."""
    g = _gen(seed, "cpu")
    total = max(N, int(round(span * N)))
    rows = []
    for _ in range(B):
        if repeats:
            r = torch.randint(0, total, (N,), generator=g).sort().values
        else:
            r = torch.randperm(total, generator=g)[:N].sort().values
        rows.append(r)
    return torch.stack(rows).to(torch.int32)
