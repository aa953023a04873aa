"""The decode with its cache split by length over ranks, end to end with the
library's kernels: 2 and 3 processes (gloo process group), all on cuda:0, each
holding its own key range of the cache.  Every rank runs ``decode_shard`` on
its keys, the parts travel through the process group's all-gather, and
``merge_lse`` combines them; every rank's result is compared with the oracle's
decode over the whole cache.  The ranks' kernels never wait on one another:
the only synchronisation between processes is the host-side all-gather.
"""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

# D, g, alpha, base, B, Hq, Hkv, shard_len, kv_len
CASES = {
    2: (128, 1, 1.0, 5e5, 3, 24, 8, 640, [1280, 700, 33]),
    3: (64, 8, 1.0, 1e6, 2, 14, 2, 500, [1500, 1001]),
}


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(world):
    from rope_wavelength_sparsity_b200 import inputs
    D, g, alpha, base, B, Hq, Hkv, shard, kv_len = CASES[world]
    q = inputs.randn_bf16((B, Hq, D), 8100 + world)
    kc = inputs.randn_bf16((B, world * shard, Hkv, D), 8200 + world)
    vc = inputs.randn_bf16((B, world * shard, Hkv, D), 8300 + world)
    return q, kc, vc


def _rank(rank, world, port, q_out):
    sys.path.insert(0, ROOT)
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import datetime
    import torch
    import torch.distributed as dist
    import rope_wavelength_sparsity_b200 as wp
    from rope_wavelength_sparsity_b200 import distributed as wd
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        D, g, alpha, base, B, Hq, Hkv, shard, kv_len = CASES[world]
        q, kc, vc = _inputs(world)
        win = wp.Window(D, base, alpha, g)
        ks = kc[:, rank * shard:(rank + 1) * shard].contiguous().cuda()
        vs = vc[:, rank * shard:(rank + 1) * shard].contiguous().cuda()
        out, lse = wd.decode_kv_split(q.cuda(), ks, vs, kv_len, win, shard_len=shard, rank=rank,
                                      world=world, scale=1 / math.sqrt(D))
        status = wp.device_status()
        q_out.put((rank, status, out.float().cpu().numpy(), lse.cpu().numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_kv_split_decode_real_kernels(cuda_dev, world):
    import oracle
    import rope_wavelength_sparsity_b200 as wp
    from rope_wavelength_sparsity_b200 import inputs
    from _parity import check_rows
    port = _free_port()
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, qq)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((qq.get(timeout=300) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    D, g, alpha, base, B, Hq, Hkv, shard, kv_len = CASES[world]
    q, kc, vc = _inputs(world)
    rows = [(b, h) for b in range(B) for h in range(Hq)]
    o_ref, l_ref = oracle.decode_rows(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len,
                                      Hq=Hq, Hkv=Hkv, base=base, alpha=alpha, g=g,
                                      scale=1 / math.sqrt(D), rows=rows)
    for rank, status, out, lse in got:
        assert status == wp.OK, rank
        check_rows(out.reshape(B * Hq, D), lse.reshape(-1), o_ref, l_ref,
                   f"rank {rank} of {world}")
    for rank in range(1, world):              # every rank holds the same merged result
        assert np.array_equal(got[0][2], got[rank][2]) and np.array_equal(got[0][3], got[rank][3])
