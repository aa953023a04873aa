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
