"""Per-RoPE-wavelength windowed causal attention for NVIDIA B200 (sm_100a).

Thin Python binding of the C ABI in ``include/wpattn.h`` (``libwpattn.so``,
built in-tree by ``rope_wavelength_sparsity_b200.build``).  The binding only
marshals arguments: tensors are passed as raw device pointers and every
step of the computation runs in the library's CUDA kernels.  There is no
fallback path: if the shared library is missing or a call fails, an
exception is raised.

Entry points (same names as the C ABI, without the ``wpattn_`` prefix):
``prefill`` (with the key-range split of ``prefill_split`` when its plan splits anything;
``prefill_split_plan``, ``prefill_split_workspace_size``), ``decode``, ``decode_pairmajor``,
``kcache_to_pairmajor``, ``decode_positions``, ``decode_paged``, ``prefill_masked``,
``pack_block_mask``, ``rope``, ``rope_qk``, ``prefill_rope``, ``decode_rope``,
``prefill_positions``, ``decode_shard``, ``merge_lse``, ``decode_workspace_size``,
``decode_noalloc``, ``pruned_fraction``, ``thresholds``, ``device_status``.

Calls are asynchronous on the given stream (torch's current stream by
default).  Every wait inside a kernel is bounded; when one runs out, the
kernel returns early, its outputs are not valid, and the only report is the
library's status word, read (and cleared) by ``device_status()``.  Callers
that need to know must poll it after their calls, or pass ``check=True`` to
``prefill``, ``decode`` or ``decode_noalloc``, which synchronises the stream
and raises ``WpattnError`` (code ``ETIMEOUT``) on a nonzero status.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwpattn.so")

OK, EINVAL, EUNSUPPORTED, ECUDA, ETIMEOUT, EWORKSPACE, EINDEX = range(7)


class WpattnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {_strerror(code)} (code {code})")


class _Window(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int32), ("group_pairs", ctypes.c_int32),
                ("rope_base", ctypes.c_double), ("alpha", ctypes.c_double)]


@dataclass(frozen=True)
class Window:
    """RoPE window: head dim D, base, factor alpha (inf = off), pair granularity g (1 or 8)."""
    head_dim: int
    rope_base: float
    alpha: float
    group_pairs: int = 1

    def _c(self) -> _Window:
        return _Window(self.head_dim, self.group_pairs, float(self.rope_base), float(self.alpha))


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded ``libwpattn.so``; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m rope_wavelength_sparsity_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
        wp = ctypes.POINTER(_Window)
        L.wpattn_thresholds.argtypes = [wp, ctypes.POINTER(ctypes.c_int64)]
        L.wpattn_pruned_fraction.argtypes = [wp, i64, i64, i64, i64,
                                             ctypes.POINTER(ctypes.c_uint64),
                                             ctypes.POINTER(ctypes.c_uint64),
                                             ctypes.POINTER(ctypes.c_double)]
        L.wpattn_prefill.argtypes = [wp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i64, i64,
                                     f32, vp]
        L.wpattn_prefill_split.argtypes = [wp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i64,
                                           i64, f32, i32, vp, ctypes.c_size_t, vp]
        L.wpattn_prefill_split_workspace_size.restype = ctypes.c_size_t
        L.wpattn_prefill_split_workspace_size.argtypes = [i32, i32, i32, i32, i32, i64, i64, i32, i32]
        L.wpattn_prefill_split_plan.argtypes = [i32, i32, i32, i32, i64, i64, i32, i32,
                                                ctypes.POINTER(ctypes.c_int64),
                                                ctypes.POINTER(ctypes.c_int32),
                                                ctypes.POINTER(ctypes.c_int32)]
        L.wpattn_prefill_masked.argtypes = [wp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i64,
                                            i64, f32, vp, i32, vp]
        L.wpattn_pack_block_mask.argtypes = [vp, vp, i64, i32, i32, vp]
        L.wpattn_prefill_positions.argtypes = [wp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp,
                                               i64, vp, i64, f32, vp]
        L.wpattn_rope.argtypes = [vp, vp, i32, i32, i32, i32, i64, vp, ctypes.c_double, vp]
        L.wpattn_rope_qk.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i64, i64,
                                     ctypes.c_double, vp]
        L.wpattn_prefill_rope.argtypes = [wp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i64, i64,
                                          f32, vp, ctypes.c_size_t, vp]
        L.wpattn_prefill_rope_workspace_size.restype = ctypes.c_size_t
        L.wpattn_prefill_rope_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
        L.wpattn_decode_workspace_size.restype = ctypes.c_size_t
        L.wpattn_decode_workspace_size.argtypes = [wp, i32, i32, i32, i64]
        L.wpattn_decode.argtypes = [wp, vp, vp, vp, ctypes.POINTER(ctypes.c_int32), i64, i32, i32,
                                    i32, f32, vp, vp, vp, ctypes.c_size_t, vp]
        L.wpattn_decode_pairmajor.argtypes = L.wpattn_decode.argtypes
        L.wpattn_kcache_to_pairmajor.argtypes = [vp, vp, i64, i32, i32, i32, vp]
        i32p = ctypes.POINTER(ctypes.c_int32)
        L.wpattn_decode_positions.argtypes = [wp, vp, vp, vp, i32p, i64, i32p, vp, i64, i32, i32,
                                              i32, f32, vp, vp, vp, ctypes.c_size_t, vp]
        L.wpattn_decode_rope.argtypes = L.wpattn_decode_positions.argtypes
        i64p = ctypes.POINTER(ctypes.c_int64)
        L.wpattn_decode_shard.argtypes = [wp, vp, vp, vp, i32p, i64, i64p, i64p, i32, i32, i32,
                                          f32, vp, vp, vp, ctypes.c_size_t, vp]
        L.wpattn_merge_lse.argtypes = [vp, vp, i32, i64, i32, vp, vp, vp]
        L.wpattn_decode_paged.argtypes = [wp, vp, vp, vp, i32, i32, vp, i32, i32p, i32p, vp, i64,
                                          i32, i32, i32, f32, vp, vp, vp, ctypes.c_size_t, vp]
        L.wpattn_device_status.argtypes = [vp]
        L.wpattn_selftest_wait_timeout.argtypes = [vp]
        L.wpattn_strerror.restype = ctypes.c_char_p
        L.wpattn_strerror.argtypes = [ctypes.c_int]
        L.wpattn_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _strerror(code: int) -> str:
    try:
        return lib().wpattn_strerror(code).decode()
    except Exception:  # pragma: no cover - only when the library itself is absent
        return "unknown"


def _check(code: int, what: str):
    if code != OK:
        raise WpattnError(code, what)


def version() -> str:
    return lib().wpattn_version().decode()


def thresholds(w: Window):
    """Per-pair thresholds T_eff[p] (list of D/2 ints; 2**63-1 = no limit)."""
    arr = (ctypes.c_int64 * (w.head_dim // 2))()
    _check(lib().wpattn_thresholds(ctypes.byref(w._c()), arr), "wpattn_thresholds")
    return list(arr)


def pruned_fraction(w: Window, Nq: int, Nk: int, q_pos0: int = 0, k_pos0: int = 0):
    """(pruned_terms, total_terms, fraction) per (batch, head) from the closed form."""
    pr, tot, fr = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_double()
    _check(lib().wpattn_pruned_fraction(ctypes.byref(w._c()), Nq, Nk, q_pos0, k_pos0,
                                        ctypes.byref(pr), ctypes.byref(tot), ctypes.byref(fr)),
           "wpattn_pruned_fraction")
    return pr.value, tot.value, fr.value


def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev_tensor(t, name):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16 or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous bf16 tensor")
    return ctypes.c_void_p(t.data_ptr())


def _shape(t, name, shape, dtype=None):
    """Check a tensor's shape (and dtype) before its pointer reaches a kernel: the C
    interface takes sizes, not buffers, so a short buffer would be read or written
    past its end."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, not {t.dtype}")


def _f32_out(t, name, shape, like):
    """An fp32 output buffer: shape, dtype, contiguity and device of `like`."""
    import torch
    _shape(t, name, shape, torch.float32)
    if not t.is_contiguous() or t.device != like.device:
        raise TypeError(f"{name} must be contiguous and on {like.device}")
    return ctypes.c_void_p(t.data_ptr())


def _prefill_shapes(q, k, v, w, out, lse):
    """(B, Nq, Hq, D, Nk, Hkv) of a prefill call, after checking that q, k, v and any
    caller-supplied out / lse agree with them and with the window's head dim."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be 4-D: [B, N, H, D]")
    B, Nq, Hq, D = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    if D != w.head_dim:
        raise ValueError(f"q has head dim {D}, the window {w.head_dim}")
    _shape(k, "k", (B, Nk, Hkv, D))
    _shape(v, "v", (B, Nk, Hkv, D))
    if out is not None:
        _shape(out, "out", q.shape)
    if lse is not None:
        _f32_out(lse, "lse", (B, Hq, Nq), q)
    return B, Nq, Hq, D, Nk, Hkv


def prefill_split_plan(B: int, Nq: int, Nk: int, Hq: int, q_pos0: int = 0, k_pos0: int = 0,
                       kv_splits: int = 0, num_sms: int = 0):
    """(main_items, split_items, parts) of ``prefill``'s key-range split: the work items
    (256-row query blocks x heads x sequences) run unsplit, those split after them, and
    the parts of each.  kv_splits 0 = the library's plan; num_sms 0 = this device."""
    m, n, s = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
    _check(lib().wpattn_prefill_split_plan(B, Nq, Nk, Hq, q_pos0, k_pos0, kv_splits, num_sms,
                                           ctypes.byref(m), ctypes.byref(n), ctypes.byref(s)),
           "wpattn_prefill_split_plan")
    return m.value, n.value, s.value


def prefill_split_workspace_size(B: int, Nq: int, Nk: int, Hq: int, D: int, q_pos0: int = 0,
                                 k_pos0: int = 0, kv_splits: int = 0, num_sms: int = 0) -> int:
    return int(lib().wpattn_prefill_split_workspace_size(B, Nq, Nk, Hq, D, q_pos0, k_pos0,
                                                         kv_splits, num_sms))


def prefill(q, k, v, w: Window, *, q_pos0: int = 0, k_pos0: int = 0, scale: float | None = None,
            out=None, lse=None, want_lse: bool = True, stream=None, check: bool = False,
            kv_splits: int | None = None, workspace=None):
    """Windowed causal prefill.  q [B,Nq,Hq,D], k/v [B,Nk,Hkv,D] bf16 CUDA tensors.

    Returns (out [B,Nq,Hq,D] bf16, lse [B,Hq,Nq] fp32 or None).  ``kv_splits``
    splits work items' key ranges into parts merged by their log-sum-exp
    (None or 0: the library's plan, ``prefill_split_plan``; 1: no split; 2..64:
    every item); a split needs ``workspace`` (uint8 CUDA, allocated here if None).
    The call is asynchronous; a kernel that gave up a bounded wait is reported
    only by ``device_status()``, unless ``check`` (synchronise and raise).
    """
    import torch
    B, Nq, Hq, D, Nk, Hkv = _prefill_shapes(q, k, v, w, out, lse)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    kv_splits = 0 if kv_splits is None else int(kv_splits)
    lse_p = ctypes.c_void_p(lse.data_ptr()) if lse is not None else None
    need = (prefill_split_workspace_size(B, Nq, Nk, Hq, D, q_pos0, k_pos0, kv_splits)
            if kv_splits != 1 and B and Nq and Nk else 0)
    if need > 0 or not 0 <= kv_splits <= 64:
        if workspace is None and need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        rc = lib().wpattn_prefill_split(ctypes.byref(w._c()), _dev_tensor(q, "q"), _dev_tensor(k, "k"),
                                        _dev_tensor(v, "v"), _dev_tensor(out, "out"), lse_p,
                                        B, Nq, Nk, Hq, Hkv, q_pos0, k_pos0,
                                        float(scale) if scale else 0.0, kv_splits,
                                        ctypes.c_void_p(workspace.data_ptr()) if workspace is not None
                                        else None, workspace.numel() if workspace is not None else 0,
                                        _stream_ptr(stream))
        _check(rc, "wpattn_prefill_split")
    else:
        rc = lib().wpattn_prefill(ctypes.byref(w._c()), _dev_tensor(q, "q"), _dev_tensor(k, "k"),
                                  _dev_tensor(v, "v"), _dev_tensor(out, "out"), lse_p,
                                  B, Nq, Nk, Hq, Hkv, q_pos0, k_pos0,
                                  float(scale) if scale else 0.0, _stream_ptr(stream))
        _check(rc, "wpattn_prefill")
    if check:
        _check(device_status(stream), "wpattn_prefill (device status)")
    return out, lse


MASK_BLOCK = 128  # rows and keys covered by one block-mask entry


def pack_block_mask(mask, stream=None):
    """Block mask [B, Hq, ceil(Nq/128), ceil(Nk/128)] (bool or uint8 CUDA, nonzero =
    attended) -> the packed bit rows ``prefill_masked`` reads: int32 [B, Hq, nqb,
    ceil(nkb/32)], bit kb % 32 of word kb // 32."""
    import torch
    if not isinstance(mask, torch.Tensor) or not mask.is_cuda or mask.dim() != 4:
        raise TypeError("mask must be a 4-D CUDA tensor")
    if mask.dtype == torch.bool:
        mask = mask.view(torch.uint8)
    if mask.dtype != torch.uint8 or not mask.is_contiguous():
        raise TypeError("mask must be a contiguous bool or uint8 tensor")
    B, Hq, nqb, nkb = mask.shape
    nw = (nkb + 31) // 32
    words = torch.empty((B, Hq, nqb, nw), dtype=torch.int32, device=mask.device)
    _check(lib().wpattn_pack_block_mask(ctypes.c_void_p(mask.data_ptr()),
                                        ctypes.c_void_p(words.data_ptr()), B * Hq * nqb, nkb, nw,
                                        _stream_ptr(stream)), "wpattn_pack_block_mask")
    return words


def prefill_masked(q, k, v, block_mask, w: Window, *, q_pos0: int = 0, k_pos0: int = 0,
                   scale: float | None = None, out=None, lse=None, want_lse: bool = True,
                   stream=None):
    """``prefill`` with a 128 x 128 block mask on top of the window and causality.

    block_mask: bool / uint8 [B, Hq, ceil(Nq/128), ceil(Nk/128)] (packed here), or the
    packed int32 words from ``pack_block_mask``.
    """
    import torch
    B, Nq, Hq, D, Nk, Hkv = _prefill_shapes(q, k, v, w, out, lse)
    if block_mask.dtype != torch.int32:
        block_mask = pack_block_mask(block_mask, stream=stream)
    nqb = (Nq + MASK_BLOCK - 1) // MASK_BLOCK
    if (block_mask.dim() != 4 or tuple(block_mask.shape[:3]) != (B, Hq, nqb)
            or not block_mask.is_cuda or not block_mask.is_contiguous()):
        raise TypeError(f"packed block mask must be a contiguous CUDA int32 [B, Hq, {nqb}, words]")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    rc = lib().wpattn_prefill_masked(ctypes.byref(w._c()), _dev_tensor(q, "q"), _dev_tensor(k, "k"),
                                     _dev_tensor(v, "v"), _dev_tensor(out, "out"),
                                     ctypes.c_void_p(lse.data_ptr()) if lse is not None else None,
                                     B, Nq, Nk, Hq, Hkv, q_pos0, k_pos0,
                                     float(scale) if scale else 0.0,
                                     ctypes.c_void_p(block_mask.data_ptr()), block_mask.shape[3],
                                     _stream_ptr(stream))
    _check(rc, "wpattn_prefill_masked")
    return out, lse


def rope(x, *, base: float, pos0: int = 0, positions=None, out=None, stream=None):
    """RoPE of x [B, N, H, D] (bf16 CUDA): pair p = dims (p, p + D/2) turns by
    pos * base^(-2p/D), token t of each sequence at pos0 + t or positions[b, t]
    (int32 CUDA [B, N]).  Rounded to bf16; ``out`` may be x."""
    import torch
    B, N, H, D = x.shape
    if out is None:
        out = torch.empty_like(x)
    _check(lib().wpattn_rope(_dev_tensor(x, "x"), _dev_tensor(out, "out"), B, N, H, D, pos0,
                             _int32_dev(positions, "positions") if positions is not None else None,
                             float(base), _stream_ptr(stream)), "wpattn_rope")
    return out


def rope_qk(q, k, *, base: float, q_pos0: int = 0, k_pos0: int = 0, q_out=None, k_out=None,
            stream=None):
    """RoPE of a prefill's q [B, Nq, Hq, D] at q_pos0 + t and k [B, Nk, Hkv, D] at
    k_pos0 + j in one launch, each as ``rope`` would turn it.  Returns (q_out, k_out)."""
    import torch
    B, Nq, Hq, D = q.shape
    if k.dim() != 4 or k.shape[0] != B or k.shape[3] != D:
        raise ValueError("k must be [B, Nk, Hkv, D] with q's B and D")
    Nk, Hkv = k.shape[1], k.shape[2]
    q_out = torch.empty_like(q) if q_out is None else q_out
    k_out = torch.empty_like(k) if k_out is None else k_out
    if tuple(q_out.shape) != tuple(q.shape) or tuple(k_out.shape) != tuple(k.shape):
        raise ValueError("q_out / k_out must have the shapes of q / k")
    _check(lib().wpattn_rope_qk(_dev_tensor(q, "q"), _dev_tensor(q_out, "q_out"), _dev_tensor(k, "k"),
                                _dev_tensor(k_out, "k_out"), B, Nq, Nk, Hq, Hkv, D, q_pos0, k_pos0,
                                float(base), _stream_ptr(stream)), "wpattn_rope_qk")
    return q_out, k_out


def prefill_rope(q, k, v, w: Window, *, q_pos0: int = 0, k_pos0: int = 0,
                 scale: float | None = None, out=None, lse=None, want_lse: bool = True,
                 workspace=None, stream=None):
    """``prefill`` from q and k before their RoPE rotation (rotated with w.rope_base at
    q_pos0 + t and k_pos0 + j into a workspace first)."""
    import torch
    B, Nq, Hq, D, Nk, Hkv = _prefill_shapes(q, k, v, w, out, lse)
    if workspace is None:
        n = int(lib().wpattn_prefill_rope_workspace_size(B, Nq, Nk, Hq, Hkv, D))
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    rc = lib().wpattn_prefill_rope(ctypes.byref(w._c()), _dev_tensor(q, "q"), _dev_tensor(k, "k"),
                                   _dev_tensor(v, "v"), _dev_tensor(out, "out"),
                                   ctypes.c_void_p(lse.data_ptr()) if lse is not None else None,
                                   B, Nq, Nk, Hq, Hkv, q_pos0, k_pos0,
                                   float(scale) if scale else 0.0,
                                   ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
                                   _stream_ptr(stream))
    _check(rc, "wpattn_prefill_rope")
    return out, lse


def prefill_positions(q, k, v, q_pos, k_pos, w: Window, *, scale: float | None = None, out=None,
                      lse=None, want_lse: bool = True, stream=None):
    """``prefill`` with explicit per-token positions: q_pos int32 CUDA [B, >= Nq], k_pos
    int32 CUDA [B, >= Nk], non-decreasing along each sequence.  k_pos is copied into a
    16-byte aligned array padded to a multiple of 128 keys when it is not one already."""
    import torch
    B, Nq, Hq, D, Nk, Hkv = _prefill_shapes(q, k, v, w, out, lse)
    _int32_dev(q_pos, "q_pos")
    _int32_dev(k_pos, "k_pos")
    padded = max(128, -(-Nk // 128) * 128)
    if (k_pos.stride(0) < padded or k_pos.stride(0) % 4 or k_pos.data_ptr() % 16
            or k_pos.shape[1] < Nk):
        kp = torch.zeros((B, padded), dtype=torch.int32, device=k_pos.device)
        kp[:, :min(Nk, k_pos.shape[1])] = k_pos[:, :Nk]
        k_pos = kp
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    rc = lib().wpattn_prefill_positions(ctypes.byref(w._c()), _dev_tensor(q, "q"), _dev_tensor(k, "k"),
                                        _dev_tensor(v, "v"), _dev_tensor(out, "out"),
                                        ctypes.c_void_p(lse.data_ptr()) if lse is not None else None,
                                        B, Nq, Nk, Hq, Hkv, ctypes.c_void_p(q_pos.data_ptr()),
                                        q_pos.stride(0), ctypes.c_void_p(k_pos.data_ptr()),
                                        k_pos.stride(0), float(scale) if scale else 0.0,
                                        _stream_ptr(stream))
    _check(rc, "wpattn_prefill_positions")
    return out, lse


def decode_workspace_size(w: Window, B: int, Hq: int, Hkv: int, max_kv_len: int) -> int:
    return int(lib().wpattn_decode_workspace_size(ctypes.byref(w._c()), B, Hq, Hkv, max_kv_len))


def _decode_shapes(q, k_cache, v_cache, kv_len, w, out, lse):
    """(B, Hq, D, L, Hkv) of a decode over a contiguous cache, after checking that the
    caches, kv_len and any caller-supplied out / lse agree with q and the window."""
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be [B, Hq, D] and k_cache [B, L, Hkv, D]")
    B, Hq, D = q.shape
    L, Hkv = k_cache.shape[1], k_cache.shape[2]
    if D != w.head_dim:
        raise ValueError(f"q has head dim {D}, the window {w.head_dim}")
    _shape(k_cache, "k_cache", (B, L, Hkv, D))
    _shape(v_cache, "v_cache", (B, L, Hkv, D))
    if len(kv_len) != B:
        raise ValueError(f"kv_len has {len(kv_len)} entries for {B} sequences")
    if out is not None:
        _shape(out, "out", q.shape)
    if lse is not None:
        _f32_out(lse, "lse", (B, Hq), q)
    return B, Hq, D, L, Hkv


def decode(q, k_cache, v_cache, kv_len, w: Window, *, scale: float | None = None, out=None,
           lse=None, want_lse: bool = True, workspace=None, stream=None, check: bool = False):
    """Windowed decode.  q [B,Hq,D]; caches [B,L,Hkv,D] bf16 CUDA; kv_len: host ints [B].

    Returns (out [B,Hq,D] bf16, lse [B,Hq] fp32 or None).  The call is
    asynchronous; a kernel that gave up a bounded wait is reported only by
    ``device_status()``, unless ``check`` (synchronise and raise).
    """
    import torch
    B, Hq, D, L, Hkv = _decode_shapes(q, k_cache, v_cache, kv_len, w, out, lse)
    kvl = (ctypes.c_int32 * B)(*[int(x) for x in kv_len])
    if workspace is None:
        n = decode_workspace_size(w, B, Hq, Hkv, L)
        if n == 0:
            raise WpattnError(EINVAL, "wpattn_decode_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    rc = lib().wpattn_decode(ctypes.byref(w._c()), _dev_tensor(q, "q"),
                             _dev_tensor(k_cache, "k_cache"), _dev_tensor(v_cache, "v_cache"),
                             kvl, L, B, Hq, Hkv, float(scale) if scale else 0.0,
                             _dev_tensor(out, "out"),
                             ctypes.c_void_p(lse.data_ptr()) if lse is not None else None,
                             ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
                             _stream_ptr(stream))
    _check(rc, "wpattn_decode")
    if check:
        _check(device_status(stream), "wpattn_decode (device status)")
    return out, lse


def kcache_to_pairmajor(k_cache, out=None, stream=None):
    """K cache [B, L, Hkv, D] -> pair-major slabs [B, Hkv, D/16, L, 16] (bf16 CUDA tensors)."""
    import torch
    B, L, Hkv, D = k_cache.shape
    if out is None:
        out = torch.empty((B, Hkv, D // 16, L, 16), dtype=k_cache.dtype, device=k_cache.device)
    _check(lib().wpattn_kcache_to_pairmajor(_dev_tensor(k_cache, "k_cache"), _dev_tensor(out, "out"),
                                            L, B, Hkv, D, _stream_ptr(stream)),
           "wpattn_kcache_to_pairmajor")
    return out


def decode_pairmajor(q, k_slabs, v_cache, kv_len, w: Window, *, scale: float | None = None,
                     out=None, lse=None, want_lse: bool = True, workspace=None, stream=None):
    """Windowed decode with K as pair-major slabs [B, Hkv, D/16, L, 16] (see
    ``kcache_to_pairmajor``); q, v_cache, kv_len and the results as for ``decode``."""
    import torch
    B, Hq, D = q.shape
    Hkv, L = k_slabs.shape[1], k_slabs.shape[3]
    kvl = (ctypes.c_int32 * B)(*[int(x) for x in kv_len])
    if workspace is None:
        n = decode_workspace_size(w, B, Hq, Hkv, L)
        if n == 0:
            raise WpattnError(EINVAL, "wpattn_decode_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    rc = lib().wpattn_decode_pairmajor(ctypes.byref(w._c()), _dev_tensor(q, "q"),
                                       _dev_tensor(k_slabs, "k_slabs"), _dev_tensor(v_cache, "v_cache"),
                                       kvl, L, B, Hq, Hkv, float(scale) if scale else 0.0,
                                       _dev_tensor(out, "out"),
                                       ctypes.c_void_p(lse.data_ptr()) if lse is not None else None,
                                       ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
                                       _stream_ptr(stream))
    _check(rc, "wpattn_decode_pairmajor")
    return out, lse


def _decode_outputs(q, w, B, Hq, Hkv, cap, out, lse, want_lse, workspace):
    import torch
    if out is not None:
        _shape(out, "out", q.shape)
    if lse is not None:
        _f32_out(lse, "lse", (B, Hq), q)
    if workspace is None:
        n = decode_workspace_size(w, B, Hq, Hkv, cap)
        if n == 0:
            raise WpattnError(EINVAL, "wpattn_decode_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    return out, lse, workspace


def _int32_dev(t, name):
    """Device pointer of a 2-D int32 CUDA tensor whose rows are contiguous."""
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.int32:
        raise TypeError(f"{name} must be an int32 CUDA tensor")
    if t.dim() != 2 or t.stride(1) != 1:
        raise TypeError(f"{name} must be 2-D with contiguous rows")
    return ctypes.c_void_p(t.data_ptr())


def decode_positions(q, k_cache, v_cache, kv_len, q_pos, k_pos, w: Window, *,
                     scale: float | None = None, out=None, lse=None, want_lse: bool = True,
                     workspace=None, stream=None):
    """Decode with explicit positions: the query of sequence b at q_pos[b] (host
    ints), cache row j at k_pos[b, j] (int32 CUDA tensor [B, >= max kv_len]).
    Caches, kv_len and results as for ``decode``."""
    B, Hq, D = q.shape
    L, Hkv = k_cache.shape[1], k_cache.shape[2]
    kvl = (ctypes.c_int32 * B)(*[int(x) for x in kv_len])
    qp = (ctypes.c_int32 * B)(*[int(x) for x in q_pos])
    out, lse, workspace = _decode_outputs(q, w, B, Hq, Hkv, L, out, lse, want_lse, workspace)
    rc = lib().wpattn_decode_positions(ctypes.byref(w._c()), _dev_tensor(q, "q"),
                                       _dev_tensor(k_cache, "k_cache"), _dev_tensor(v_cache, "v_cache"),
                                       kvl, L, qp, _int32_dev(k_pos, "k_pos"), k_pos.stride(0), B,
                                       Hq, Hkv, float(scale) if scale else 0.0, _dev_tensor(out, "out"),
                                       ctypes.c_void_p(lse.data_ptr()) if lse is not None else None,
                                       ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
                                       _stream_ptr(stream))
    _check(rc, "wpattn_decode_positions")
    return out, lse


def decode_rope(q, k_cache, v_cache, kv_len, w: Window, *, q_pos=None, k_pos=None,
                scale: float | None = None, out=None, lse=None, want_lse: bool = True,
                workspace=None, stream=None):
    """``decode`` (or ``decode_positions``) with q before its RoPE rotation; the kernel
    turns q by its position with w.rope_base as it loads it."""
    B, Hq, D = q.shape
    L, Hkv = k_cache.shape[1], k_cache.shape[2]
    kvl = (ctypes.c_int32 * B)(*[int(x) for x in kv_len])
    qp = (ctypes.c_int32 * B)(*[int(x) for x in q_pos]) if q_pos is not None else None
    out, lse, workspace = _decode_outputs(q, w, B, Hq, Hkv, L, out, lse, want_lse, workspace)
    rc = lib().wpattn_decode_rope(ctypes.byref(w._c()), _dev_tensor(q, "q"),
                                  _dev_tensor(k_cache, "k_cache"), _dev_tensor(v_cache, "v_cache"),
                                  kvl, L, qp,
                                  _int32_dev(k_pos, "k_pos") if k_pos is not None else None,
                                  k_pos.stride(0) if k_pos is not None else 0, B, Hq, Hkv,
                                  float(scale) if scale else 0.0, _dev_tensor(out, "out"),
                                  ctypes.c_void_p(lse.data_ptr()) if lse is not None else None,
                                  ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
                                  _stream_ptr(stream))
    _check(rc, "wpattn_decode_rope")
    return out, lse


def decode_shard(q, k_shard, v_shard, kv_len, q_pos, k_pos0, w: Window, *,
                 scale: float | None = None, out=None, lse=None, workspace=None, stream=None):
    """Decode over one length-shard of a cache: the query of sequence b at q_pos[b], the
    shard's keys at k_pos0[b] + j for j < kv_len[b] (host ints; kv_len may be 0).  Returns
    (out normalised over the shard's keys, lse) for ``merge_lse``."""
    import torch
    B, Hq, D = q.shape
    L, Hkv = k_shard.shape[1], k_shard.shape[2]
    kvl = (ctypes.c_int32 * B)(*[int(x) for x in kv_len])
    qp = (ctypes.c_int64 * B)(*[int(x) for x in q_pos])
    kp = (ctypes.c_int64 * B)(*[int(x) for x in k_pos0])
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    out, lse, workspace = _decode_outputs(q, w, B, Hq, Hkv, L, out, lse, True, workspace)
    rc = lib().wpattn_decode_shard(ctypes.byref(w._c()), _dev_tensor(q, "q"),
                                   _dev_tensor(k_shard, "k_shard"), _dev_tensor(v_shard, "v_shard"),
                                   kvl, L, qp, kp, B, Hq, Hkv, float(scale) if scale else 0.0,
                                   _dev_tensor(out, "out"), ctypes.c_void_p(lse.data_ptr()),
                                   ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
                                   _stream_ptr(stream))
    _check(rc, "wpattn_decode_shard")
    return out, lse


def merge_lse(outs, lses, *, out=None, lse=None, stream=None):
    """Combine parts outs [R, ..., D] (bf16 CUDA) with their lses [R, ...] (fp32 CUDA)
    into (out [..., D], lse [...])."""
    import torch
    R, D = outs.shape[0], outs.shape[-1]
    rows = outs[0].numel() // D
    if lses.dtype != torch.float32 or not lses.is_cuda or not lses.is_contiguous():
        raise TypeError("lses must be a contiguous fp32 CUDA tensor")
    if out is None:
        out = torch.empty(outs.shape[1:], dtype=outs.dtype, device=outs.device)
    if lse is None:
        lse = torch.empty(lses.shape[1:], dtype=torch.float32, device=outs.device)
    _check(lib().wpattn_merge_lse(_dev_tensor(outs, "outs"), ctypes.c_void_p(lses.data_ptr()), R,
                                  rows, D, _dev_tensor(out, "out"), ctypes.c_void_p(lse.data_ptr()),
                                  _stream_ptr(stream)), "wpattn_merge_lse")
    return out, lse


def decode_paged(q, k_pages, v_pages, block_table, kv_len, w: Window, *, q_pos=None, k_pos=None,
                 scale: float | None = None, out=None, lse=None, want_lse: bool = True,
                 workspace=None, stream=None):
    """Decode from page pools k_pages, v_pages [num_pages, page_size, Hkv, D] (bf16
    CUDA) through block_table (int32 CUDA [B, max_pages_per_seq]); optional
    explicit positions as for ``decode_positions``.  Results as for ``decode``."""
    B, Hq, D = q.shape
    num_pages, page_size, Hkv = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    if not block_table.is_contiguous():
        raise TypeError("block_table must be contiguous")
    max_pages = block_table.shape[1]
    kvl = (ctypes.c_int32 * B)(*[int(x) for x in kv_len])
    qp = (ctypes.c_int32 * B)(*[int(x) for x in q_pos]) if q_pos is not None else None
    out, lse, workspace = _decode_outputs(q, w, B, Hq, Hkv, max_pages * page_size, out, lse,
                                          want_lse, workspace)
    rc = lib().wpattn_decode_paged(ctypes.byref(w._c()), _dev_tensor(q, "q"),
                                   _dev_tensor(k_pages, "k_pages"), _dev_tensor(v_pages, "v_pages"),
                                   num_pages, page_size, _int32_dev(block_table, "block_table"),
                                   max_pages, kvl, qp,
                                   _int32_dev(k_pos, "k_pos") if k_pos is not None else None,
                                   k_pos.stride(0) if k_pos is not None else 0, B, Hq, Hkv,
                                   float(scale) if scale else 0.0, _dev_tensor(out, "out"),
                                   ctypes.c_void_p(lse.data_ptr()) if lse is not None else None,
                                   ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
                                   _stream_ptr(stream))
    _check(rc, "wpattn_decode_paged")
    return out, lse


def decode_noalloc(q, k_cache, v_cache, kv_len, w: Window, *, scale: float | None = None,
                   out=None, lse=None, want_lse: bool = True, stream=None, check: bool = False):
    """Decode with the library's built-in scratch instead of a workspace.

    For callers that cannot allocate device memory at the call site; the
    problem's partial results must fit the built-in array
    (``decode_noalloc_max_bytes()``), calls on one device share it.  With
    ``check`` the stream is synchronised and a nonzero device status raises.
    """
    import torch
    B, Hq, D, L, Hkv = _decode_shapes(q, k_cache, v_cache, kv_len, w, out, lse)
    kvl = (ctypes.c_int32 * B)(*[int(x) for x in kv_len])
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    fn = lib().wpattn_decode_noalloc
    fn.argtypes = [ctypes.POINTER(_Window), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.POINTER(ctypes.c_int32), ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                   ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_void_p]
    rc = fn(ctypes.byref(w._c()), _dev_tensor(q, "q"), _dev_tensor(k_cache, "k_cache"),
            _dev_tensor(v_cache, "v_cache"), kvl, L, B, Hq, Hkv, float(scale) if scale else 0.0,
            _dev_tensor(out, "out"), ctypes.c_void_p(lse.data_ptr()) if lse is not None else None,
            _stream_ptr(stream))
    _check(rc, "wpattn_decode_noalloc")
    if check:
        _check(device_status(stream), "wpattn_decode_noalloc (device status)")
    return out, lse


def decode_noalloc_max_bytes() -> int:
    fn = lib().wpattn_decode_noalloc_max_bytes
    fn.restype = ctypes.c_size_t
    return int(fn())


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the kernels' status word."""
    return int(lib().wpattn_device_status(_stream_ptr(stream)))


def selftest_wait_timeout(stream=None) -> None:
    """Launch the library's bounded-wait self-check: one kernel waits on a
    barrier nothing arrives at until its 2 s bound runs out, then records
    WPATTN_ETIMEOUT for the next ``device_status``."""
    _check(lib().wpattn_selftest_wait_timeout(_stream_ptr(stream)), "wpattn_selftest_wait_timeout")


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
