"""Oracle for per-RoPE-wavelength windowed causal attention (test infrastructure).

Only the tests, the package's ``smoke()`` check and the CPU-baseline leg of
``bench.py`` may import this module.  The product path (the CUDA library and
its Python binding) never does, and the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, double precision, one thread);
this module compiles it with the host C compiler on first use and exposes
numpy-friendly wrappers.  Each wrapper names the passage it follows; see the
header of ``oracle.c`` for the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

T_INF = (1 << 63) - 1


def build() -> str:
    """Compile oracle.c into a shared object (idempotent)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not os.path.exists(_LIB_PATH)
            or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64p = ctypes.POINTER(ctypes.c_int64)
            u64p = ctypes.POINTER(ctypes.c_uint64)
            dp = ctypes.POINTER(ctypes.c_double)
            vp = ctypes.c_void_p
            lib.oracle_thresholds.argtypes = [ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                              ctypes.c_int, i64p, dp]
            lib.oracle_attention_rows.argtypes = [
                vp, vp, vp, vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                ctypes.c_double, ctypes.c_int, ctypes.c_double, ctypes.c_int64, vp, vp, vp]
            lib.oracle_scores.argtypes = [vp, vp, ctypes.c_int64, ctypes.c_int, ctypes.c_int64,
                                          ctypes.c_int64, ctypes.c_double, ctypes.c_double,
                                          ctypes.c_int, vp]
            lib.oracle_attention_rows_masked.argtypes = [
                vp, vp, vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                ctypes.c_double, ctypes.c_int, ctypes.c_double, vp, ctypes.c_int64,
                ctypes.c_int64, ctypes.c_int64, vp, vp, vp]
            lib.oracle_rope.argtypes = [vp, vp, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_double, vp, vp]
            lib.oracle_attention_positions.argtypes = [
                vp, vp, vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, vp, ctypes.c_int64, vp, ctypes.c_int64,
                ctypes.c_double, ctypes.c_double, ctypes.c_int, ctypes.c_double, ctypes.c_int64,
                vp, vp, vp]
            lib.oracle_decode_positions.argtypes = [
                vp, vp, vp, vp, vp, vp, ctypes.c_int64, ctypes.c_int, ctypes.c_int64,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double,
                ctypes.c_int, ctypes.c_double, ctypes.c_int64, vp, vp, vp]
            for name in ("oracle_count_bruteforce", "oracle_count_rows"):
                getattr(lib, name).argtypes = [ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                               ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                               ctypes.c_int64, ctypes.c_int64, u64p, u64p]
            _lib = lib
    return _lib


def _u16(a: np.ndarray) -> np.ndarray:
    """bf16 payload as a contiguous uint16 array (accepts uint16 or torch bf16 bits)."""
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are raw bf16 bit patterns (uint16)")
    return a


def thresholds(D: int, base: float, alpha: float, g: int):
    """T_eff[p] per pair and the smallest distance of alpha*lambda_p to an integer.

    ATFlash Abstract ("wavelength-proportional distance"), WavePrune Original
    abstract (first rotation period at alpha = 1, 16-dim blocks for g = 8).
    """
    lib = _load()
    T = np.zeros(D // 2, dtype=np.int64)
    margin = ctypes.c_double(0.0)
    rc = lib.oracle_thresholds(D, base, alpha, g,
                               T.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                               ctypes.byref(margin))
    if rc != 0:
        raise ValueError("oracle_thresholds: bad arguments")
    return T, margin.value


def attention_rows(q, k, v, *, Hq, Hkv, q_pos0=0, k_pos0=0, base, alpha, g, scale,
                   rows, kv_len=None):
    """out [n, D] and lse [n] (float64) for the (b, h, t) triples in ``rows``.

    q: uint16 [B, Nq, Hq, D]; k, v: uint16 [B, Nk, Hkv, D] (bf16 bit patterns).
    ATFlash Abstract: windowed score, unchanged softmax.
    """
    lib = _load()
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, Nq, _, D = q.shape
    Nk = k.shape[1]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    kvl = None
    if kv_len is not None:
        kvl = np.ascontiguousarray(np.asarray(kv_len, dtype=np.int64))
    rc = lib.oracle_attention_rows(
        q.ctypes.data, k.ctypes.data, v.ctypes.data,
        kvl.ctypes.data if kvl is not None else None,
        B, Nq, Nk, Hq, Hkv, D, q_pos0, k_pos0, base, alpha, g, scale, n,
        rows.ctypes.data, out.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_attention_rows failed ({rc})")
    return out, lse


def attention_rows_masked(q, k, v, block_mask, *, Hq, Hkv, q_pos0=0, k_pos0=0, base, alpha, g,
                          scale, rows, block_q=128, block_k=128):
    """As ``attention_rows``, with key j of row t attended only where
    block_mask[b, h, t // block_q, j // block_k] is nonzero.

    block_mask: [B, Hq, ceil(Nq / block_q), ceil(Nk / block_k)], any integer or
    bool dtype.  ATFlash Abstract: the window composes with token selection.
    """
    lib = _load()
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, Nq, _, D = q.shape
    Nk = k.shape[1]
    nqb, nkb = -(-Nq // block_q), -(-Nk // block_k)
    m = np.ascontiguousarray(np.asarray(block_mask) != 0, dtype=np.uint8)
    if m.shape != (B, Hq, nqb, nkb):
        raise ValueError(f"block_mask shape {m.shape}, want {(B, Hq, nqb, nkb)}")
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    rc = lib.oracle_attention_rows_masked(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, B, Nq, Nk, Hq, Hkv, D, q_pos0, k_pos0,
        base, alpha, g, scale, m.ctypes.data, block_q, block_k, n, rows.ctypes.data,
        out.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_attention_rows_masked failed ({rc})")
    return out, lse


def attention_positions(q, k, v, q_pos, k_pos, *, Hq, Hkv, base, alpha, g, scale, rows):
    """Prefill rows with explicit positions: query t of sequence b at q_pos[b, t], key j at
    k_pos[b, j] (int arrays [B, >= Nq] and [B, >= Nk]); otherwise as ``attention_rows``.
    ATFlash Abstract: the window depends on the relative position only.
    """
    lib = _load()
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, Nq, _, D = q.shape
    Nk = k.shape[1]
    qp = np.ascontiguousarray(np.asarray(q_pos, dtype=np.int64).reshape(B, -1))
    kp = np.ascontiguousarray(np.asarray(k_pos, dtype=np.int64).reshape(B, -1))
    if qp.shape[1] < Nq or kp.shape[1] < Nk:
        raise ValueError("position arrays shorter than the sequences")
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    rc = lib.oracle_attention_positions(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, B, Nq, Nk, Hq, Hkv, D, qp.ctypes.data,
        qp.shape[1], kp.ctypes.data, kp.shape[1], base, alpha, g, scale, n, rows.ctypes.data,
        out.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_attention_positions failed ({rc})")
    return out, lse


def decode_rows(q, k_cache, v_cache, kv_len, *, Hq, Hkv, base, alpha, g, scale, rows=None):
    """Decode: one new query per sequence at position kv_len[b]-1 over keys 0..kv_len[b]-1.

    q: uint16 [B, Hq, D]; caches uint16 [B, Lmax, Hkv, D].  Same definition as
    ``attention_rows`` with Nq = 1 and a per-sequence key count.
    """
    q = _u16(q)
    B, _, D = q.shape
    kv_len = np.asarray(kv_len, dtype=np.int64)
    if rows is None:
        rows = [(b, h) for b in range(B) for h in range(Hq)]
    outs, lses = [], []
    for (b, h) in rows:
        # each sequence has its own query position, so rows go one at a time
        qb = q[b:b + 1].reshape(1, 1, Hq, D)
        o, l = attention_rows(qb, k_cache[b:b + 1], v_cache[b:b + 1], Hq=Hq, Hkv=Hkv,
                              q_pos0=int(kv_len[b]) - 1, k_pos0=0, base=base, alpha=alpha,
                              g=g, scale=scale, rows=[(0, h, 0)], kv_len=kv_len[b:b + 1])
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.array(lses)


def decode_positions(q, k_cache, v_cache, kv_len, q_pos, k_pos, *, Hq, Hkv, base, alpha, g,
                     scale, rows=None):
    """Decode with explicit positions: the query of sequence b sits at q_pos[b] and
    its key j < kv_len[b] at k_pos[b, j]; keys past the query are excluded.

    q: uint16 [B, Hq, D]; caches uint16 [B, Lmax, Hkv, D]; k_pos int [B, >= max kv_len].
    ATFlash Abstract: the window is a function of the relative position q_pos - k_pos.
    """
    lib = _load()
    q, k_cache, v_cache = _u16(q), _u16(k_cache), _u16(v_cache)
    B, _, D = q.shape
    Lmax = k_cache.shape[1]
    kvl = np.ascontiguousarray(np.asarray(kv_len, dtype=np.int64).reshape(B))
    qp = np.ascontiguousarray(np.asarray(q_pos, dtype=np.int64).reshape(B))
    kp = np.ascontiguousarray(np.asarray(k_pos, dtype=np.int64).reshape(B, -1))
    if kp.shape[1] < int(kvl.max(initial=0)):
        raise ValueError("k_pos has fewer columns than the longest sequence")
    if rows is None:
        rows = [(b, h) for b in range(B) for h in range(Hq)]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
    n = rows.shape[0]
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    rc = lib.oracle_decode_positions(
        q.ctypes.data, k_cache.ctypes.data, v_cache.ctypes.data, kvl.ctypes.data,
        qp.ctypes.data, kp.ctypes.data, kp.shape[1], B, Lmax, Hq, Hkv, D, base, alpha, g,
        scale, n, rows.ctypes.data, out.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_decode_positions failed ({rc})")
    return out, lse


def rope(x, positions, *, base, exact=False):
    """RoPE of bf16 vectors x [n, H, D] (uint16 bits), token i at positions[i].

    Pair p = dims (p, p + D/2) turns by positions[i] * base^(-2p/D) (WavePrune,
    Original abstract).  Returns uint16 bf16 bits rounded to nearest-even from the
    exact result, or with ``exact`` the float64 result itself.
    """
    lib = _load()
    x = _u16(x)
    n, H, D = x.shape
    pos = np.ascontiguousarray(np.asarray(positions, dtype=np.int64).reshape(n))
    if exact:
        out = np.zeros((n, H, D), dtype=np.float64)
        rc = lib.oracle_rope(x.ctypes.data, pos.ctypes.data, n, H, D, base, None, out.ctypes.data)
    else:
        out = np.zeros((n, H, D), dtype=np.uint16)
        rc = lib.oracle_rope(x.ctypes.data, pos.ctypes.data, n, H, D, base, out.ctypes.data, None)
    if rc != 0:
        raise ValueError("oracle_rope: bad arguments")
    return out


def scores(qrow, keys, *, q_pos, k_pos0=0, base, alpha, g):
    """Windowed scores (no scale) of one query row vs keys [n, D]; NaN = causal."""
    lib = _load()
    qrow, keys = _u16(qrow), _u16(keys)
    n, D = keys.shape
    s = np.zeros(n, dtype=np.float64)
    rc = lib.oracle_scores(qrow.ctypes.data, keys.ctypes.data, n, D, q_pos, k_pos0,
                           base, alpha, g, s.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_scores failed")
    return s


def _count(fn, D, base, alpha, g, Nq, Nk, q_pos0, k_pos0):
    pr = ctypes.c_uint64(0)
    tot = ctypes.c_uint64(0)
    rc = fn(D, base, alpha, g, Nq, Nk, q_pos0, k_pos0, ctypes.byref(pr), ctypes.byref(tot))
    if rc != 0:
        raise ValueError("oracle count: bad arguments")
    return pr.value, tot.value


def count_bruteforce(D, base, alpha, g, Nq, Nk, q_pos0=0, k_pos0=0):
    """(pruned, total) pair-terms per (batch, head) by full enumeration (tiny sizes)."""
    return _count(_load().oracle_count_bruteforce, D, base, alpha, g, Nq, Nk, q_pos0, k_pos0)


def count_rows(D, base, alpha, g, Nq, Nk, q_pos0=0, k_pos0=0):
    """(pruned, total) pair-terms per (batch, head), one query row at a time.

    ATFlash Abstract: the reduction rate is input-independent and has a
    closed form in N.
    """
    return _count(_load().oracle_count_rows, D, base, alpha, g, Nq, Nk, q_pos0, k_pos0)
