"""Decode with the KV cache split by length across devices, one process per GPU.

Rank r holds keys [r * shard_len, (r + 1) * shard_len) of every sequence (a
contiguous range of the cache, in its own memory).  Each rank attends the
query to its own keys with ``decode_shard`` (result normalised over those
keys, plus their log-sum-exp); one all-gather then gives every rank the
parts of every other rank, and ``merge_lse`` combines them into the decode
over the whole cache.  The exchange is (D + 2) values per (sequence, query
head) per rank.  No rank reads another rank's memory.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence


def shard_keys(kv_len_total: Sequence[int], rank: int, shard_len: int):
    """(k_pos0, kv_len) of rank ``rank``'s shard: its first key position and how
    many keys of each sequence it holds (0 when the sequence ends before it)."""
    start = rank * shard_len
    k_pos0 = [start for _ in kv_len_total]
    kv_len = [max(0, min(shard_len, int(n) - start)) for n in kv_len_total]
    return k_pos0, kv_len


def _all_gather(t, world: int, group=None):
    """[world, *t.shape] stack of every rank's t, in rank order, on t's device.
    Moved as raw bytes so that any backend carries bf16 bit for bit; the gloo
    backend, which gathers host tensors only, goes through a host copy."""
    import torch
    import torch.distributed as dist
    src = t.contiguous().view(torch.uint8)
    staged = src.is_cuda and dist.get_backend(group) == "gloo"
    if staged:
        src = src.cpu()
    parts = [torch.empty_like(src) for _ in range(world)]
    dist.all_gather(parts, src, group=group)
    out = torch.stack(parts)
    if staged:
        out = out.to(t.device)
    return out.view(t.dtype)


def decode_kv_split(q, k_shard, v_shard, kv_len_total: Sequence[int], w, *, shard_len: int,
                    rank: int, world: int, group=None, scale: Optional[float] = None,
                    shard_fn: Optional[Callable] = None, merge_fn: Optional[Callable] = None):
    """Decode of q [B, Hq, D] against a cache whose sequence b has kv_len_total[b]
    keys, of which this rank holds [rank * shard_len, ...) in k_shard, v_shard
    [B, shard_len, Hkv, D].  The query of sequence b sits at kv_len_total[b] - 1.
    Returns (out [B, Hq, D], lse [B, Hq]) on every rank.

    ``shard_fn`` / ``merge_fn`` default to the library's ``decode_shard`` and
    ``merge_lse`` (the only compute); they are parameters so that the exchange
    logic can be exercised with other implementations of the same contract.
    """
    import rope_wavelength_sparsity_b200 as wp
    k_pos0, kv_len = shard_keys(kv_len_total, rank, shard_len)
    q_pos = [int(n) - 1 for n in kv_len_total]
    if shard_fn is None:
        def shard_fn(q_, k_, v_, kv_len_, q_pos_, k_pos0_, w_, scale_):
            return wp.decode_shard(q_, k_, v_, kv_len_, q_pos_, k_pos0_, w_, scale=scale_)
    if merge_fn is None:
        def merge_fn(outs_, lses_):
            return wp.merge_lse(outs_, lses_)
    out_r, lse_r = shard_fn(q, k_shard, v_shard, kv_len, q_pos, k_pos0, w, scale)
    if world == 1:
        return merge_fn(out_r.unsqueeze(0), lse_r.unsqueeze(0))
    outs = _all_gather(out_r, world, group)
    lses = _all_gather(lse_r, world, group)
    return merge_fn(outs, lses)
