"""The benchmark's multi-rank path on CPU ranks (gloo, world size 2).

Each rank runs an independent problem (weak scaling); the only collective
is the max-over-ranks of the step time.  These tests run that reduction and
the whole-job throughput arithmetic as two gloo processes, and check that
the reference arm does its work on rank 0 only.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
        mx = bench._max_over_ranks(local_ms, world)
        val = bench.weak_scaling_value(2.0e12, world, mx)
        q.put((rank, mx, val))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, val in got:
        assert mx == 15.0                                # every rank sees the slowest rank
        assert val == pytest.approx(2 * 2.0e12 / 15.0e-3)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class A:
        workload, steps, warmup = "tiny", 1, 1
    rank, res = bench.reference_arm(A())
    assert rank == 1 and res is None


# ---------------------------------------------------------------------------
# decode with the cache split by length over ranks: the exchange and merge
# logic of rope_wavelength_sparsity_b200.distributed on two gloo ranks, with
# the oracle standing in for the per-shard kernel (CPU only) and a numpy merge
# ---------------------------------------------------------------------------

def _oracle_shard(q, k_, v_, kv_len, q_pos, k_pos0, win, scale):
    import numpy as np
    import torch
    import oracle
    from rope_wavelength_sparsity_b200 import inputs
    B, Hq, D = q.shape
    L = k_.shape[1]
    kp = np.array([[k_pos0[b] + j for j in range(L)] for b in range(B)], dtype=np.int64)
    o, l = oracle.decode_positions(inputs.bits(q), inputs.bits(k_), inputs.bits(v_), kv_len, q_pos,
                                   kp, Hq=Hq, Hkv=k_.shape[2], base=win.rope_base,
                                   alpha=win.alpha, g=win.group_pairs, scale=scale)
    out = torch.tensor(o.reshape(B, Hq, D), dtype=torch.float32).to(torch.bfloat16)
    return out, torch.tensor(l.reshape(B, Hq), dtype=torch.float32)


def _numpy_merge(outs, lses):
    import numpy as np
    import torch
    o = outs.float().numpy().astype(np.float64)
    l = lses.numpy().astype(np.float64)
    M = l.max(axis=0)
    with np.errstate(invalid="ignore"):
        w = np.where(np.isneginf(l), 0.0, np.exp(l - M))
    W = w.sum(axis=0)
    out = np.where(W[..., None] > 0, (w[..., None] * o).sum(axis=0) / np.maximum(W, 1e-300)[..., None], 0.0)
    lse = np.where(W > 0, M + np.log(np.maximum(W, 1e-300)), -np.inf)
    return torch.tensor(out), torch.tensor(lse)


def _split_worker(rank, world, port, q_out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import datetime
    import torch.distributed as dist
    import rope_wavelength_sparsity_b200 as wp
    from rope_wavelength_sparsity_b200 import inputs
    from rope_wavelength_sparsity_b200 import distributed as wd
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, Hq, Hkv, D, shard = 3, 4, 2, 16, 40
        kv_len = [80, 23, 41]                 # sequence 1 ends inside rank 0's shard
        q = inputs.randn_bf16((B, Hq, D), 601)
        kc = inputs.randn_bf16((B, world * shard, Hkv, D), 602)
        vc = inputs.randn_bf16((B, world * shard, Hkv, D), 603)
        win = wp.Window(D, 100.0, 1.0, 1)
        ks = kc[:, rank * shard:(rank + 1) * shard].contiguous()
        vs = vc[:, rank * shard:(rank + 1) * shard].contiguous()
        out, lse = wd.decode_kv_split(q, ks, vs, kv_len, win, shard_len=shard, rank=rank,
                                      world=world, scale=0.25, shard_fn=_oracle_shard,
                                      merge_fn=_numpy_merge)
        q_out.put((rank, out.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


def test_decode_kv_split_exchange_gloo():
    import numpy as np
    import oracle
    import rope_wavelength_sparsity_b200 as wp
    from rope_wavelength_sparsity_b200 import inputs
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, qq)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((qq.get(timeout=120) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, Hq, Hkv, D, shard = 3, 4, 2, 16, 40
    kv_len = [80, 23, 41]
    q = inputs.randn_bf16((B, Hq, D), 601)
    kc = inputs.randn_bf16((B, world * shard, Hkv, D), 602)
    vc = inputs.randn_bf16((B, world * shard, Hkv, D), 603)
    o_ref, l_ref = oracle.decode_rows(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), kv_len,
                                      Hq=Hq, Hkv=Hkv, base=100.0, alpha=1.0, g=1, scale=0.25)
    for rank, out, lse in got:                   # every rank holds the whole result
        np.testing.assert_allclose(out.reshape(-1, D), o_ref, atol=1e-2)   # parts travel as bf16
        np.testing.assert_allclose(lse.reshape(-1), l_ref, atol=1e-5)
    assert np.array_equal(got[0][1], got[1][1])


def test_shard_keys_bounds():
    from rope_wavelength_sparsity_b200 import distributed as wd
    assert wd.shard_keys([100, 30, 0], 0, 40) == ([0, 0, 0], [40, 30, 0])
    assert wd.shard_keys([100, 30, 0], 1, 40) == ([40, 40, 40], [40, 0, 0])
    assert wd.shard_keys([100, 30, 0], 2, 40) == ([80, 80, 80], [20, 0, 0])


def test_reference_arm_loads_no_product_library():
    """The oracle arm (``--impl reference``) counts its work with the oracle and loads
    nothing from the library: run it in a fresh process and read that process's
    mapped files."""
    import json
    import subprocess
    code = (
        "import json, sys\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        "import bench\n"
        "class A:\n"
        "    workload, steps, warmup, ref_seconds = 'tiny', 1, 1, 0.5\n"
        "rank, res = bench.reference_arm(A())\n"
        "maps = open('/proc/self/maps').read()\n"
        "print(json.dumps({'res': res, 'wpattn': 'libwpattn' in maps,\n"
        "                  'oracle': 'liboracle' in maps}))\n")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                         timeout=600, env={**os.environ, "WORLD_SIZE": "1", "RANK": "0"})
    assert out.returncode == 0, out.stderr[-2000:]
    got = json.loads(out.stdout.strip().splitlines()[-1])
    assert got["oracle"] and not got["wpattn"]
    res = got["res"]
    assert res["impl"] == "reference" and res["value"] > 0
    assert res["config"]["workload"] == "tiny" and res["config"]["Nk"] == 256
    assert res["cpu_baseline"]["cores"] >= 1 and res["cpu_baseline"]["kind"] == "oracle"
    # the whole tiny step at the measured rate, its work counted with the oracle
    import bench
    from rope_wavelength_sparsity_b200 import inputs
    full = bench.full_step_work_oracle(inputs.WORKLOADS["tiny"])
    assert res["ms_per_step"] == pytest.approx(full / (res["value"] * 1e12) * 1e3, rel=1e-3)
