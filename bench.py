"""Benchmark of per-RoPE-wavelength windowed attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one pass of the hot path over one batch of synthetic input: the
host planner (thresholds, tile plan) and the windowed prefill kernel of the
chosen workload, called through the C ABI.  The default workload is the
largest single-GPU one: the Qwen2.5-7B-1M-shaped prefill of the last 16384
queries against 1,048,576 causal keys (Hq=28, Hkv=4, D=128, base 1e7,
alpha 1, g = 8 pairs).  The same run times the other workloads as nested
objects under "configs", each with its roofline, window-off speedup and
end-to-end figure: the Qwen2.5-0.5B-shaped 32K prefill (with the block-mask,
pre-RoPE and explicit-positions variants), the Llama-3.2-3B-shaped 128K
prefill at alpha 1 and 2, and the Llama-3.2-3B-shaped (B=16, L=128K) and
Qwen2.5-7B-shaped (B=1, L=1M) decodes with their pair-major and paged
layouts.

Metric: effective TFLOP/s = (4 * kept QK pair-terms + 2 * D * causal
(query, key) pairs) per (batch, query head), over the device time of the
step; decode: algorithmic GB/s = K bytes of the kept pairs + all V bytes
(+ q and out) over the decode call's device time.

Timing: CUDA events on the launching stream around every step, an L2 flush
(a 512 MiB write, then a read of 256 MiB of it, so that the flush's own dirty
lines are written back before the step rather than inside it) between steps
outside the events, W warm-up steps, barrier
+ synchronize around the timed region, max over ranks.  Multi-GPU: every rank
runs its own independent problem (weak scaling, no data-path collective).

``--impl reference`` times the oracle (the plain CPU definition) on a bounded
sample of rows of the same workload, in the same metric, on the host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import itertools
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "effective TFLOP/s (kept QK terms + PV) and decode KV GB/s, % of B200 roofline"
DEFAULT_WORKLOAD = "qwen2.5-7b-1m-prefill"
# the other workloads, timed as nested objects of the default line
NESTED_PREFILL = ("qwen2.5-0.5b-32k", "llama3.2-3b-128k-a1", "llama3.2-3b-128k-a2")
NESTED_DECODE = ("llama3.2-3b-decode-128k", "qwen2.5-7b-1m-decode")
# the block-mask, pre-RoPE and explicit-positions variants run on this one
VARIANTS_WORKLOAD = "qwen2.5-0.5b-32k"
FLUSH_BYTES = 512 << 20
FLUSH_NOTE = ("flushed between steps (512 MiB write, then a 256 MiB read of it: no dirty "
              "line of the flush is written back inside a step)")

# DRAM bytes (read + write) per launch of a workload's dominant kernel from one
# ncu capture, keyed by workload and by a hash of that kernel's sources (code
# only: comments and layout do not count) at capture time: a changed kernel
# reports null until it is captured again.
NCU_TRAFFIC = {
    # prefill_kernel<128, 1, 0, 0, 0> on the full 1M-key chunk, its 1,776 unsplit items (one
    # pass): 57.86 GB read + 128.71 MB written; K and V (2.15 GB) come from DRAM about 27 times,
    # at 4-5 % of the HBM bandwidth (43.5 to 59.8 GB over captures of this grid: the CTAs' drift
    # along their walks decides how much an L2 line is shared)
    ("qwen2.5-7b-1m-prefill", "86ede3d69d7a58b8"): 57860000000 + 128710000,
    # prefill_kernel<64, 1, 0, 0, 0> on the Qwen2.5-0.5B 32K prefill (one pass): 75.60 MB read +
    # 21.47 MB written, against 75.5 MB of inputs and 60.5 MB of outputs (part of the output is
    # still in L2 when the kernel ends)
    ("qwen2.5-0.5b-32k", "86ede3d69d7a58b8"): 75600000 + 21470000,
    # decode_split_kernel<128, 3, 0> on the full B=16, L=131072 Llama decode (one pass):
    # 8.59 GB read + 3.66 MB written (all of K and V: whole rows of the [B, L, Hkv, D] cache)
    ("llama3.2-3b-decode-128k", "3e21e0f2bf8b391e"): 8590000000 + 3660000,
}

KERNEL_SOURCES = {"prefill": ("prefill_kernel.cuh", "device_util.cuh"),
                  "decode": ("decode_kernels.cuh", "device_util.cuh", "rope_kernels.cuh")}


def _code_only(text: str) -> str:
    """Source text without comments and with whitespace runs collapsed: a change of a
    comment or of layout alone leaves the kernel (and its counters) as they were."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "rope_wavelength_sparsity_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            pk = json.load(fh)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk.get("bf16_tflops_sustained"), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def workload_config(w, world: int) -> dict:
    """The `config` object of a workload's line (the same for both arms)."""
    if w.kind == "prefill":
        return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
                "Nq": w.Nq, "Nk": w.Nk, "q_pos0": w.q_pos0, "rope_base": w.base,
                "alpha": w.alpha, "group_pairs": w.g, "global_batch": w.B * world,
                "seq_len": w.Nk, "parallelism": f"independent problem per GPU x{world}",
                "l2": FLUSH_NOTE}
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "L": w.Nk,
            "rope_base": w.base, "alpha": w.alpha, "group_pairs": w.g,
            "global_batch": w.B * world, "seq_len": w.Nk,
            "parallelism": f"independent problem per GPU x{world}",
            "l2": FLUSH_NOTE}


# ----------------------------------------------------------- work accounting
def prefill_flops(w, win, wp):
    """(effective FLOPs, window-off FLOPs) of one prefill of workload w."""
    pruned, total, _ = wp.pruned_fraction(win, w.Nq, w.Nk, w.q_pos0, w.k_pos0)
    P = w.D // 2
    causal = total // P
    kept = total - pruned
    per_head = 4 * kept + 2 * w.D * causal
    off = 4 * w.D * causal
    return w.B * w.Hq * per_head, w.B * w.Hq * off


def masked_flops(w, win, wp, mask):
    """Effective FLOPs of one prefill under a block mask (bool [B, Hq, nqb, nkb], 128 x 128
    blocks): the kept QK pair-terms and PV of the causal (query, key) pairs of each attended
    block, counted block by block with the closed-form count."""
    P, blk = w.D // 2, wp.MASK_BLOCK
    cache = {}
    total = 0
    for idx in mask.nonzero().tolist():
        qb, kb = idx[2], idx[3]
        nq = min(blk, w.Nq - qb * blk)
        nk = min(blk, w.Nk - kb * blk)
        key = (nq, nk, w.q_pos0 + qb * blk - (w.k_pos0 + kb * blk))
        if key not in cache:
            pr, tot, _ = wp.pruned_fraction(win, nq, nk, key[2], 0)
            cache[key] = 4 * (tot - pr) + 2 * w.D * (tot // P)
        total += cache[key]
    return total


def decode_bytes(w, win, wp, kv_len):
    """(algorithmic bytes, window-off bytes) of one decode step."""
    P = w.D // 2
    kbytes = vbytes = kfull = 0
    for L in kv_len:
        pruned, total, _ = wp.pruned_fraction(win, 1, L, L - 1, 0)
        kept = total - pruned
        kbytes += kept * 2 * 2 * w.Hkv
        kfull += total * 2 * 2 * w.Hkv
        vbytes += L * w.D * 2 * w.Hkv
    io = w.B * w.Hq * w.D * 2 * 2 + w.B * w.Hq * 4
    return kbytes + vbytes + io, kfull + vbytes + io


def row_flops_oracle(w, t):
    """Effective FLOPs of prefill query row t of workload w, counted with the oracle's
    own row-wise count (so that the oracle arm shares no code with the product)."""
    import oracle
    pruned, total = oracle.count_rows(w.D, w.base, w.alpha, w.g, 1, w.Nk, w.q_pos0 + t,
                                      w.k_pos0)
    P = w.D // 2
    return 4 * (total - pruned) + 2 * w.D * (total // P)


def decode_row_bytes_oracle(w, L):
    """Algorithmic bytes of one decode (sequence, query head) row over L keys, counted with
    the oracle's row-wise count: the group's K slice and V, shared by its G query heads."""
    import oracle
    pruned, total = oracle.count_rows(w.D, w.base, w.alpha, w.g, 1, L, L - 1, 0)
    return ((total - pruned) * 4 + L * w.D * 2) / (w.Hq // w.Hkv)


def full_step_work_oracle(w, kv_len=None):
    """Effective FLOPs (prefill) or algorithmic bytes (decode, sequences of kv_len keys) of
    one whole step of workload w, counted with the oracle's own pair-term count."""
    import oracle
    P = w.D // 2
    if w.kind == "prefill":
        pruned, total = oracle.count_rows(w.D, w.base, w.alpha, w.g, w.Nq, w.Nk, w.q_pos0,
                                          w.k_pos0)
        return w.B * w.Hq * (4 * (total - pruned) + 2 * w.D * (total // P))
    return sum(w.Hq * decode_row_bytes_oracle(w, int(L)) for L in (kv_len or [w.Nk] * w.B))


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        # raw samples: $WPATTN_CLOCK_DIR if set (to keep them), else the temp directory
        out_dir = os.environ.get("WPATTN_CLOCK_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"wpattn_clocks_rank{device_index}_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not os.environ.get("WPATTN_CLOCK_DIR"):
            try:
                os.remove(self.path)
            except OSError:
                pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- GPU arm
def _dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def _max_over_ranks(x: float, world: int) -> float:
    """Largest value over all ranks (the timing reduction; no data-path collective)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, world: int, max_ms_per_step: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's step time."""
    return world * units_per_rank / (max_ms_per_step * 1e-3)


def _barrier(world):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def time_steps(step, n_warm, n_steps, flush, world, clocks=None):
    """Device time (ms) of n_steps calls of step(); L2 flushed before each.
    Returns (max over ranks of the summed step times, per-step times, clock record)."""
    import torch
    for _ in range(n_warm):
        flush()
        step()
    _barrier(world)
    if clocks:
        clocks.start()
        time.sleep(0.25)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(n_steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(n_steps)]
    for i in range(n_steps):
        flush()
        starts[i].record()
        step()
        ends[i].record()
    _barrier(world)
    clk = clocks.stop() if clocks else None
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return _max_over_ranks(sum(per), world), per, clk


def _tensor_peak(peaks, clk, timed_ms):
    """(peak TFLOP/s, label): the sustained GEMM figure for a kernel timed over a long
    region (at least a second) under the power cap (its clock samples saw
    sw_power_cap), else the burst one.  A short run that only inherits the cap flag
    from the run before it is held against the burst figure."""
    capped = bool(clk) and "sw_power_cap" in (clk.get("reasons") or [])
    if capped and timed_ms >= 1000.0 and peaks.get("bf16_tflops_sustained"):
        return peaks["bf16_tflops_sustained"], f"{peaks['source']} bf16 dense (sustained, sw_power_cap active)"
    return peaks["bf16_tflops"], f"{peaks['source']} bf16 dense (burst)"


# ex2.approx issue rate of one SM (4 per clock per sub-partition; measured with a probe
# of independent chains, 8 cycles per warp instruction at 1, 2 and 4 warps per SP)
EXP_PER_CLK_SM = 16


def exp_roof(w, off_flops, kernel_ms, clk, dev):
    """Second roof of a prefill step: every causal (query, key) score needs one exponential
    on the special-function unit, whatever the window prunes.  Its peak comes from the unit
    count and the maximum SM clock; floor_ms is the step time at that rate."""
    import torch
    exps = off_flops // (4 * w.D)        # window-off FLOPs = 4 D per causal pair and head
    mhz = (clk or {}).get("sm_max_mhz") or 1965.0
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    peak = EXP_PER_CLK_SM * sms * mhz * 1e6
    floor_ms = exps / peak * 1e3
    return {"bound": "mufu", "exps_per_step": int(exps), "peak": peak, "unit": "exp/s",
            "achieved": round(exps / (kernel_ms * 1e-3), 1), "floor_ms": round(floor_ms, 3),
            "frac": round(floor_ms / kernel_ms, 4),
            "peak_source": f"{EXP_PER_CLK_SM}/clk/SM x {sms} SMs x {mhz:.0f} MHz"}


def _check_status(wp, what):
    if wp.device_status() != wp.OK:
        raise RuntimeError(f"{what}: kernel status not ok")


def bench_prefill(w, args, world, rank, dev, flush, peaks, variants=False):
    """One prefill workload: the windowed call, the same call with the window off, and
    the end-to-end call with host buffers; with ``variants`` also the block-mask,
    pre-RoPE and explicit-positions variants of the same problem."""
    import torch
    import rope_wavelength_sparsity_b200 as wp
    from rope_wavelength_sparsity_b200 import inputs
    win = wp.Window(w.D, w.base, w.alpha, w.g)
    win_off = wp.Window(w.D, w.base, float("inf"), w.g)
    q, k, v, _ = inputs.prefill_inputs(w, seed=rank, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    eff, off_flops = prefill_flops(w, win, wp)
    # the library's key-range split plan for this grid, its workspace made once
    main_items, split_items, parts = wp.prefill_split_plan(w.B, w.Nq, w.Nk, w.Hq, w.q_pos0, w.k_pos0)
    S = 0 if split_items else 1
    nws = wp.prefill_split_workspace_size(w.B, w.Nq, w.Nk, w.Hq, w.D, w.q_pos0, w.k_pos0, 0)
    ws = torch.empty(nws, dtype=torch.uint8, device=dev) if split_items else None
    # the prefill kernel; with a split, the split items' kernel and their merge
    launches = (1 if main_items else 0) + (2 if split_items else 0)

    def step():
        wp.prefill(q, k, v, win, q_pos0=w.q_pos0, k_pos0=w.k_pos0, scale=w.scale, out=out, lse=lse,
                   kv_splits=S, workspace=ws)

    def step_off():
        wp.prefill(q, k, v, win_off, q_pos0=w.q_pos0, k_pos0=w.k_pos0, scale=w.scale, out=out,
                   lse=lse, kv_splits=S, workspace=ws)

    def step_unsplit():
        wp.prefill(q, k, v, win, q_pos0=w.q_pos0, k_pos0=w.k_pos0, scale=w.scale, out=out, lse=lse,
                   kv_splits=1)

    clocks = ClockSampler(dev.index) if rank == 0 else None
    total_ms, per, clk = time_steps(step, args.warmup, args.steps, flush, world, clocks)
    _check_status(wp, w.name)
    n_off = max(3, args.steps // 4)
    off_ms, _, _ = time_steps(step_off, args.warmup, n_off, flush, world)
    _check_status(wp, w.name + " window off")
    ms_step = total_ms / args.steps
    off_ms_step = off_ms / n_off
    unsplit = None
    if split_items:
        un_ms, _, _ = time_steps(step_unsplit, 1, n_off, flush, world)
        _check_status(wp, w.name + " unsplit")
        unsplit = {"ms_per_step": round(un_ms / n_off, 4),
                   "speedup_of_split": round((un_ms / n_off) / ms_step, 3)}
    kernel_ms = statistics.mean(per)
    achieved = eff / (kernel_ms * 1e-3) / 1e12
    peak_t, peak_label = _tensor_peak(peaks, clk, total_ms)
    res = {
        "metric": METRIC, "value": round(weak_scaling_value(eff, world, ms_step) / 1e12, 2),
        "unit": "TFLOP/s", "ms_per_step": round(ms_step, 4), "dtype": "bf16",
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak_t,
                     "unit": "TFLOP/s", "frac": round(achieved / peak_t, 4),
                     "traffic": NCU_TRAFFIC.get((w.name, kernel_source_hash("prefill"))),
                     "peak_source": peak_label},
        "window_off": {"ms_per_step": round(off_ms_step, 4),
                       "speedup": round(off_ms_step / ms_step, 3),
                       "ideal_speedup": round(off_flops / eff, 3),
                       "effective_tflops_at_window_off_time": round(eff / (off_ms_step * 1e-3) / 1e12, 2)},
        "work": {"effective_tflop_per_step": round(world * eff / 1e12, 4),
                 "window_off_tflop_per_step": round(world * off_flops / 1e12, 4),
                 "pruned_fraction": wp.pruned_fraction(win, w.Nq, w.Nk, w.q_pos0, w.k_pos0)[2]},
        "split_plan": {"unsplit_items": main_items, "split_items": split_items,
                       "parts_per_split_item": parts},
        "gpu_launches": launches * args.steps,
        "clocks": clk,
        "config": workload_config(w, world),
    }
    if unsplit:
        res["unsplit"] = unsplit
    res["exp_roof"] = exp_roof(w, off_flops, kernel_ms, clk, dev)
    if variants:
        res.update(_prefill_variants(w, args, world, rank, dev, flush, peaks, q, k, v, out, lse,
                                     win, eff, ms_step))
    # end to end through the public API with pinned host buffers
    qh = q.cpu().pin_memory()
    kh = k.cpu().pin_memory()
    vh = v.cpu().pin_memory()
    oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def step_e2e():
        qd = q.copy_(qh, non_blocking=True)
        kd = k.copy_(kh, non_blocking=True)
        vd = v.copy_(vh, non_blocking=True)
        o, _ = wp.prefill(qd, kd, vd, win, q_pos0=w.q_pos0, k_pos0=w.k_pos0, scale=w.scale,
                          out=out, lse=lse, kv_splits=S, workspace=ws)
        oh.copy_(o, non_blocking=True)

    n_e2e = max(5, args.steps // 4)
    e2e_ms, _, _ = time_steps(step_e2e, 2, n_e2e, flush, world)
    _check_status(wp, w.name + " end to end")
    res["e2e"] = {"value": round(world * eff / (e2e_ms / n_e2e * 1e-3) / 1e12, 2),
                  "unit": "TFLOP/s", "h2d_bytes_per_step": (q.numel() + k.numel() + v.numel()) * 2,
                  "d2h_bytes_per_step": out.numel() * 2,
                  "inputs": "all of q, k and v copied every step"}
    # A chunk far into a context (keys before the chunk's first query): the earlier keys'
    # K and V were written by the earlier chunks and stay resident, as a decode's KV cache
    # does; each step copies the chunk's q and its own k and v rows.
    new0 = max(0, w.q_pos0 - w.k_pos0)
    if 0 < new0 < w.Nk:
        kd_new = [k[b, new0:] for b in range(w.B)]
        vd_new = [v[b, new0:] for b in range(w.B)]
        kh_new = [kh[b, new0:] for b in range(w.B)]
        vh_new = [vh[b, new0:] for b in range(w.B)]

        def step_e2e_chunk():
            q.copy_(qh, non_blocking=True)
            for b in range(w.B):
                kd_new[b].copy_(kh_new[b], non_blocking=True)
                vd_new[b].copy_(vh_new[b], non_blocking=True)
            o, _ = wp.prefill(q, k, v, win, q_pos0=w.q_pos0, k_pos0=w.k_pos0, scale=w.scale,
                              out=out, lse=lse, kv_splits=S, workspace=ws)
            oh.copy_(o, non_blocking=True)

        c_ms, _, _ = time_steps(step_e2e_chunk, 2, n_e2e, flush, world)
        _check_status(wp, w.name + " end to end, chunk inputs")
        new_rows = w.Nk - new0
        res["e2e_chunk_inputs"] = {
            "value": round(world * eff / (c_ms / n_e2e * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": (q.numel() + 2 * w.B * new_rows * w.Hkv * w.D) * 2,
            "d2h_bytes_per_step": out.numel() * 2,
            "inputs": f"q and the chunk's own {new_rows} k and v rows per sequence; the "
                      f"{new0} earlier keys' K and V resident on the device"}
        del kd_new, vd_new, kh_new, vh_new
    del q, k, v, out, lse, qh, kh, vh, oh, ws
    torch.cuda.empty_cache()
    return res


def _prefill_variants(w, args, world, rank, dev, flush, peaks, q, k, v, out, lse, win, eff,
                      ms_step):
    """Block-mask, pre-RoPE and explicit-positions calls of the same prefill problem."""
    import torch
    import rope_wavelength_sparsity_b200 as wp
    from rope_wavelength_sparsity_b200 import inputs
    res = {}
    n_v = max(3, args.steps // 2)
    # the same call under a MInference-shaped block mask (vertical + slash tiles)
    mask = inputs.vertical_slash_mask(w.B, w.Hq, w.Nq, w.Nk, seed=rank, q_pos0=w.q_pos0,
                                      k_pos0=w.k_pos0)
    words = wp.pack_block_mask(mask.to(dev))
    m_eff = masked_flops(w, win, wp, mask)

    def step_masked():
        wp.prefill_masked(q, k, v, words, win, q_pos0=w.q_pos0, k_pos0=w.k_pos0, scale=w.scale,
                          out=out, lse=lse)

    m_ms, m_per, _ = time_steps(step_masked, args.warmup, n_v, flush, world)
    _check_status(wp, "masked prefill")
    m_ach = m_eff / (statistics.mean(m_per) * 1e-3) / 1e12
    causal_tiles = sum(1 for qb in range(mask.shape[2]) for kb in range(mask.shape[3])
                       if kb * 128 + w.k_pos0 <= w.q_pos0 + qb * 128 + 127)
    res["block_sparse"] = {
        "value": round(weak_scaling_value(m_eff, world, m_ms / n_v) / 1e12, 2),
        "unit": "TFLOP/s", "ms_per_step": round(m_ms / n_v, 4),
        "roofline": {"bound": "tensor", "achieved": round(m_ach, 2), "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": round(m_ach / peaks["bf16_tflops"], 4),
                     "traffic": None},
        "speedup_vs_unmasked": round(ms_step / (m_ms / n_v), 3),
        "ideal_speedup": round(eff / m_eff, 3),
        "attended_tile_fraction": round(float(mask.sum()) / (w.B * w.Hq * causal_tiles), 4),
        "mask": "vertical-slash: sink + 3 random key tiles per head, 16-tile diagonal band",
        "gpu_launches": n_v,
    }
    del words, mask
    # the same prefill from pre-RoPE q and k: rotation pre-pass + attention, and the
    # rotation kernel alone (HBM-bound: read and write q and k once)
    ws_r = torch.empty(max(1, int(wp.lib().wpattn_prefill_rope_workspace_size(
        w.B, w.Nq, w.Nk, w.Hq, w.Hkv, w.D))), dtype=torch.uint8, device=dev)
    qr_buf = torch.empty_like(q)
    kr_buf = torch.empty_like(k)

    def step_rope_prefill():
        wp.prefill_rope(q, k, v, win, q_pos0=w.q_pos0, k_pos0=w.k_pos0, scale=w.scale, out=out,
                        lse=lse, workspace=ws_r)

    def step_rope_only():
        wp.rope_qk(q, k, base=w.base, q_pos0=w.q_pos0, k_pos0=w.k_pos0, q_out=qr_buf, k_out=kr_buf)

    rp_ms, _, _ = time_steps(step_rope_prefill, args.warmup, n_v, flush, world)
    ro_ms, ro_per, _ = time_steps(step_rope_only, args.warmup, n_v, flush, world)
    _check_status(wp, "rope kernels")
    rope_bytes = 2 * 2 * (q.numel() + k.numel())
    ro_gbs = rope_bytes / (statistics.mean(ro_per) * 1e-3) / 1e9
    res["rope"] = {
        "prefill_from_prerope": {"ms_per_step": round(rp_ms / n_v, 4),
                                 "value": round(weak_scaling_value(eff, world, rp_ms / n_v) / 1e12, 2),
                                 "unit": "TFLOP/s",
                                 "overhead_vs_prefill": round((rp_ms / n_v) / ms_step - 1.0, 4),
                                 "gpu_launches": 2 * n_v},
        "rotation_kernels": {"ms_per_step": round(ro_ms / n_v, 4),
                             "roofline": {"bound": "hbm", "achieved": round(ro_gbs, 1),
                                          "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                          "frac": round(ro_gbs / peaks["hbm_gbs"], 4),
                                          "traffic": None},
                             "bytes_per_step": rope_bytes, "gpu_launches": n_v},
    }
    del ws_r, qr_buf, kr_buf
    # the same prefill through the explicit-positions kernel, given the workload's own
    # contiguous positions (same work; the cost of the searched column ranges)
    qp = (w.q_pos0 + torch.arange(w.Nq, dtype=torch.int32, device=dev)).repeat(w.B, 1)
    kp = (w.k_pos0 + torch.arange(w.Nk, dtype=torch.int32, device=dev)).repeat(w.B, 1)

    def step_pos():
        wp.prefill_positions(q, k, v, qp, kp, win, scale=w.scale, out=out, lse=lse)

    pos_ms, pos_per, _ = time_steps(step_pos, args.warmup, n_v, flush, world)
    _check_status(wp, "positions prefill")
    pos_ach = eff / (statistics.mean(pos_per) * 1e-3) / 1e12
    res["explicit_positions"] = {
        "value": round(weak_scaling_value(eff, world, pos_ms / n_v) / 1e12, 2),
        "unit": "TFLOP/s", "ms_per_step": round(pos_ms / n_v, 4),
        "roofline": {"bound": "tensor", "achieved": round(pos_ach, 2), "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": round(pos_ach / peaks["bf16_tflops"], 4),
                     "traffic": None},
        "slowdown_vs_plain": round((pos_ms / n_v) / ms_step, 3),
        "positions": "the workload's contiguous positions passed as int32 arrays",
        "gpu_launches": n_v,
    }
    del qp, kp
    return res


def bench_decode(w, args, world, rank, dev, flush, peaks):
    """One decode workload: the contiguous-cache call, window off, pair-major and paged
    layouts of the same cache, and the end-to-end call with the query from the host."""
    import torch
    import rope_wavelength_sparsity_b200 as wp
    from rope_wavelength_sparsity_b200 import inputs
    win = wp.Window(w.D, w.base, w.alpha, w.g)
    win_off = wp.Window(w.D, w.base, float("inf"), w.g)
    q, kc, vc, kv_len = inputs.decode_inputs(w, seed=rank, device=dev)
    kv_len = [int(x) for x in kv_len]
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(wp.decode_workspace_size(win, w.B, w.Hq, w.Hkv, w.Nk), dtype=torch.uint8,
                     device=dev)
    alg, off_bytes = decode_bytes(w, win, wp, kv_len)

    def step():
        wp.decode(q, kc, vc, kv_len, win, scale=w.scale, out=out, lse=lse, workspace=ws)

    def step_off():
        wp.decode(q, kc, vc, kv_len, win_off, scale=w.scale, out=out, lse=lse, workspace=ws)

    steps = args.steps
    clocks = ClockSampler(dev.index) if rank == 0 else None
    total_ms, per, clk = time_steps(step, args.warmup, steps, flush, world, clocks)
    _check_status(wp, w.name)
    n_off = max(3, steps // 4)
    off_ms, _, _ = time_steps(step_off, args.warmup, n_off, flush, world)
    _check_status(wp, w.name + " window off")
    ms = total_ms / steps
    off_step = off_ms / n_off
    achieved = alg / (statistics.mean(per) * 1e-3) / 1e9
    res = {
        "metric": METRIC, "value": round(weak_scaling_value(alg, world, ms) / 1e9, 1), "unit": "GB/s",
        "ms_per_step": round(ms, 4), "dtype": "bf16",
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "traffic": NCU_TRAFFIC.get((w.name, kernel_source_hash("decode"))),
                     "peak_source": f"{peaks['source']} HBM copy",
                     "timed": "split + combine kernels (one decode call)"},
        "window_off": {"ms_per_step": round(off_step, 4), "speedup": round(off_step / ms, 3),
                       "ideal_speedup": round(off_bytes / alg, 3)},
        "work": {"algorithmic_bytes_per_step": alg * world, "window_off_bytes_per_step": off_bytes * world},
        "gpu_launches": 2 * steps,
        "clocks": clk,
        "config": workload_config(w, world),
    }
    # the same call with K in the pair-major layout (converted once, outside the timed region):
    # the window then also cuts the bytes K moves from HBM
    slabs = wp.kcache_to_pairmajor(kc)

    def step_pm():
        wp.decode_pairmajor(q, slabs, vc, kv_len, win, scale=w.scale, out=out, lse=lse, workspace=ws)

    pm_ms, pm_per, _ = time_steps(step_pm, args.warmup, steps, flush, world)
    _check_status(wp, "pair-major decode")
    pm_achieved = alg / (statistics.mean(pm_per) * 1e-3) / 1e9
    res["pairmajor"] = {
        "value": round(weak_scaling_value(alg, world, pm_ms / steps) / 1e9, 1), "unit": "GB/s",
        "ms_per_step": round(pm_ms / steps, 4),
        "roofline": {"bound": "hbm", "achieved": round(pm_achieved, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(pm_achieved / peaks["hbm_gbs"], 4),
                     "traffic": None, "peak_source": f"{peaks['source']} HBM copy"},
        "speedup_vs_window_off": round(off_step / (pm_ms / steps), 3),
        "layout": "K [B, Hkv, D/16, L, 16] pair-major slabs, V [B, L, Hkv, D]",
        "gpu_launches": 2 * steps,
    }
    del slabs
    # the same call from a paged cache (16-row pages in shuffled pool order, the page size
    # serving engines default to), scattered once outside the timed region
    page = 16
    table, num_pages = inputs.page_layout(kv_len, page, seed=rank + 100)
    kp = inputs.scatter_to_pages(kc, kv_len, table, page, num_pages)
    vp = inputs.scatter_to_pages(vc, kv_len, table, page, num_pages)
    table = table.to(dev)
    ws_pg = torch.empty(wp.decode_workspace_size(win, w.B, w.Hq, w.Hkv, table.shape[1] * page),
                        dtype=torch.uint8, device=dev)

    def step_pg():
        wp.decode_paged(q, kp, vp, table, kv_len, win, scale=w.scale, out=out, lse=lse,
                        workspace=ws_pg)

    pg_ms, pg_per, _ = time_steps(step_pg, args.warmup, steps, flush, world)
    _check_status(wp, "paged decode")
    pg_achieved = alg / (statistics.mean(pg_per) * 1e-3) / 1e9
    res["paged"] = {
        "value": round(weak_scaling_value(alg, world, pg_ms / steps) / 1e9, 1), "unit": "GB/s",
        "ms_per_step": round(pg_ms / steps, 4),
        "roofline": {"bound": "hbm", "achieved": round(pg_achieved, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(pg_achieved / peaks["hbm_gbs"], 4),
                     "traffic": None, "peak_source": f"{peaks['source']} HBM copy"},
        "layout": f"K, V page pools [{num_pages}, {page}, Hkv, D], shuffled block table",
        "gpu_launches": 2 * steps,
    }
    del kp, vp, ws_pg
    if world > 1 and getattr(args, "kv_split", False):
        # strong scaling: the same decode (rank 0's problem) with its cache split by
        # length; each rank holds L / world keys of every sequence
        from rope_wavelength_sparsity_b200 import distributed as wd
        q0, kc0, vc0, kvl0 = inputs.decode_inputs(w, seed=0, device=dev)
        kvl0 = [int(x) for x in kvl0]
        shard = (w.Nk + world - 1) // world
        ks = kc0[:, rank * shard:(rank + 1) * shard].contiguous()
        vs = vc0[:, rank * shard:(rank + 1) * shard].contiguous()
        del kc0, vc0
        alg0, _ = decode_bytes(w, win, wp, kvl0)

        def step_split():
            wd.decode_kv_split(q0, ks, vs, kvl0, win, shard_len=shard, rank=rank, world=world,
                               scale=w.scale)

        sp_ms, _, _ = time_steps(step_split, args.warmup, steps, flush, world)
        res["kv_split"] = {
            "value": round(alg0 / (sp_ms / steps * 1e-3) / 1e9, 1), "unit": "GB/s",
            "ms_per_step": round(sp_ms / steps, 4), "scaling": "strong",
            "exchange": "one all-gather of (out, lse) parts per step, then merge_lse",
        }
        del ks, vs
    qh = q.cpu().pin_memory()
    oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def step_e2e():
        qd = q.copy_(qh, non_blocking=True)
        o, _ = wp.decode(qd, kc, vc, kv_len, win, scale=w.scale, out=out, lse=lse, workspace=ws)
        oh.copy_(o, non_blocking=True)

    n_e2e = max(5, steps // 4)
    e2e_ms, _, _ = time_steps(step_e2e, 2, n_e2e, flush, world)
    _check_status(wp, w.name + " end to end")
    res["e2e"] = {"value": round(world * alg / (e2e_ms / n_e2e * 1e-3) / 1e9, 1), "unit": "GB/s",
                  "h2d_bytes_per_step": q.numel() * 2, "d2h_bytes_per_step": out.numel() * 2,
                  "note": "the KV cache is resident on the device, as in serving"}
    del q, kc, vc, out, lse, ws
    torch.cuda.empty_cache()
    return res


def _run_workload(name, args, world, rank, dev, flush, peaks):
    from rope_wavelength_sparsity_b200 import inputs
    w = inputs.WORKLOADS[name]
    if w.kind == "prefill":
        return bench_prefill(w, args, world, rank, dev, flush, peaks,
                             variants=(name == VARIANTS_WORKLOAD and not args.only_primary))
    return bench_decode(w, args, world, rank, dev, flush, peaks)


def gpu_arm(args):
    import torch
    from rope_wavelength_sparsity_b200 import inputs

    world, rank, local = _dist_setup(args)
    dev = torch.device("cuda", local if world > 1 else 0)
    peaks = load_peaks()
    w = inputs.WORKLOADS[args.workload]
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    flush_words = flush_buf[: FLUSH_BYTES // 2].view(torch.int32)

    def flush():
        # the write evicts every line of the step's inputs; the read then
        # replaces the write's dirty lines with clean ones, so their write-back
        # is not charged to the next step
        flush_buf.fill_(1)
        flush_words.sum()

    result = _run_workload(args.workload, args, world, rank, dev, flush, peaks)
    if args.workload == DEFAULT_WORKLOAD and not args.only_primary:
        result["configs"] = {name: _run_workload(name, args, world, rank, dev, flush, peaks)
                             for name in NESTED_PREFILL + NESTED_DECODE}
    result.update({"n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                   "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                   "data": "synthetic (seeded N(0,1) bf16; pair magnitudes / planted key per workload)"})
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, time_budget_s=args.cpu_seconds)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return rank, result


# --------------------------------------------------------- oracle (CPU) arm
def host_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover - non-Linux hosts
        return os.cpu_count() or 1


def oracle_sample(w, n_rows, seed=0):
    """Rows of a workload spread over heads and positions: (b, h, t) for a prefill,
    (b, h) for a decode."""
    import numpy as np
    rng = np.random.default_rng(seed)
    rows = []
    if w.kind == "prefill":
        for i in range(n_rows):
            rows.append((0, i % w.Hq, int(rng.integers(0, w.Nq))))
    else:
        for i in range(n_rows):
            rows.append((i % w.B, (i * 7) % w.Hq))
    return rows


class _OracleJob:
    """The oracle on one sampled row at a time, with each row's work counted by the
    oracle's own pair-term count before any timing starts."""

    def __init__(self, w, n_rows):
        import torch
        import oracle
        from rope_wavelength_sparsity_b200 import inputs
        self.w = w
        self.oracle = oracle
        # inputs are drawn on the GPU when there is one (only to generate them quickly)
        gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
        self.rows = oracle_sample(w, n_rows)
        if w.kind == "prefill":
            q, k, v, _ = inputs.prefill_inputs(w, seed=0, device=gen_dev)
            self.work = [row_flops_oracle(w, t) for (_, _, t) in self.rows]
            self.unit, self.scale = "TFLOP/s", 1e12
        else:
            q, k, v, kv_len = inputs.decode_inputs(w, seed=0, device=gen_dev)
            self.kv_len = [int(x) for x in kv_len]
            self.work = [decode_row_bytes_oracle(w, self.kv_len[b]) for (b, _) in self.rows]
            self.unit, self.scale = "GB/s", 1e9
        self.qb, self.kb, self.vb = inputs.bits(q), inputs.bits(k), inputs.bits(v)
        del q, k, v

    def run(self, i):
        w, r = self.w, self.rows[i]
        if w.kind == "prefill":
            self.oracle.attention_rows(self.qb, self.kb, self.vb, Hq=w.Hq, Hkv=w.Hkv,
                                       q_pos0=w.q_pos0, k_pos0=w.k_pos0, base=w.base,
                                       alpha=w.alpha, g=w.g, scale=w.scale, rows=[r])
        else:
            self.oracle.decode_rows(self.qb, self.kb, self.vb, self.kv_len, Hq=w.Hq, Hkv=w.Hkv,
                                    base=w.base, alpha=w.alpha, g=w.g, scale=w.scale, rows=[r])

    def timed(self, budget_s, threads):
        """(value, rows done, seconds): rows taken in order by ``threads`` host threads
        until the budget is spent (the oracle's C code runs outside the GIL)."""
        counter = itertools.count()
        lock = threading.Lock()
        done = []

        def worker(t_end):
            while time.perf_counter() < t_end:
                with lock:
                    i = next(counter)
                if i >= len(self.rows):
                    return
                self.run(i)
                with lock:
                    done.append(i)

        t0 = time.perf_counter()
        ths = [threading.Thread(target=worker, args=(t0 + budget_s,)) for _ in range(threads)]
        for th in ths:
            th.start()
        for th in ths:
            th.join()
        dt = time.perf_counter() - t0
        work = sum(self.work[i] for i in done)
        return work / dt / self.scale, len(done), dt


def cpu_baseline(w, time_budget_s=15.0):
    """The oracle timed on the host on a bounded sample of the workload: on all the
    host's cores (independent rows, one per thread) and on one core."""
    cores = host_cores()
    job = _OracleJob(w, n_rows=max(4096, 64 * cores))
    what = "query rows (random heads/positions)" if w.kind == "prefill" else "(sequence, head) rows"
    measure = ("effective FLOPs of those rows / wall time" if w.kind == "prefill" else
               "algorithmic bytes of those rows (per-head share of the group's K/V) / wall time")
    one, n1, t1 = job.timed(time_budget_s, 1)
    allc, na, ta = job.timed(time_budget_s, cores)
    return {"value": round(allc, 6), "unit": job.unit, "cores": cores, "kind": "oracle",
            "sample": f"{na} {what} of {w.name} on {cores} threads, {ta:.1f} s; {measure}; "
                      "work counted with the oracle's own pair-term count",
            "one_core": {"value": round(one, 6), "unit": job.unit, "cores": 1,
                         "sample": f"{n1} rows of the same sample, {t1:.1f} s"}}


def reference_arm(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return rank, None
    from rope_wavelength_sparsity_b200 import inputs
    w = inputs.WORKLOADS[args.workload]
    cores = host_cores()
    # about 90 s of oracle work in all (--ref-seconds), spread over the steps
    per_step = max(0.2, getattr(args, "ref_seconds", 90.0) / max(1, args.steps + args.warmup))
    job = _OracleJob(w, n_rows=max(4096, 64 * cores))
    vals = []
    rows_done = 0
    for i in range(args.warmup + args.steps):
        val, n, _ = job.timed(per_step, cores)
        if i >= args.warmup:
            vals.append(val)
            rows_done += n
    value = statistics.mean(vals) if vals else 0.0
    # the whole workload's step at that rate (its work counted with the oracle's own count)
    full = full_step_work_oracle(w, getattr(job, "kv_len", None))
    ms_step = full / (value * job.scale) * 1e3 if value > 0 else None
    sample = (f"each step: rows of {w.name} on {cores} threads for {per_step:.1f} s "
              f"({rows_done} rows over the timed steps); work counted with the oracle's own "
              "pair-term count; ms_per_step is the whole workload's step at the measured rate")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": job.unit,
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(ms_step, 3) if ms_step else None,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": workload_config(w, world),
           "cpu_baseline": {"value": value, "unit": job.unit, "cores": cores, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": job.unit, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    return rank, out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only-primary", action="store_true",
                    help="time only the chosen workload (no nested configs or variants)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="oracle time budget of each cpu_baseline figure (1 core, all cores)")
    ap.add_argument("--ref-seconds", type=float, default=90.0,
                    help="--impl reference: oracle time over all its steps")
    ap.add_argument("--kv-split", action="store_true",
                    help="with N > 1: also time each decode with its cache split by length over "
                         "the ranks (strong scaling, one all-gather per step)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        rank, res = reference_arm(args)
    else:
        rank, res = gpu_arm(args)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
