"""The binding's argument checks (CPU, no kernel runs).

The C interface takes pointers and sizes, so the Python binding checks that
every tensor it hands over has the shape the sizes imply; a short buffer
would otherwise be read or written past its end on the device.  Consistent
CPU tensors pass every shape check and stop at the device check instead.
"""
import pytest
import torch

import rope_wavelength_sparsity_b200 as wp


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


WIN = wp.Window(64, 1e4, 1.0, 1)


def test_prefill_consistent_shapes_reach_the_device_check():
    q, k, v = _bf16(1, 10, 4, 64), _bf16(1, 12, 2, 64), _bf16(1, 12, 2, 64)
    with pytest.raises(TypeError, match="CUDA"):
        wp.prefill(q, k, v, WIN)
    lse = torch.zeros((1, 4, 10), dtype=torch.float32)
    with pytest.raises(TypeError, match="CUDA"):
        wp.prefill(q, k, v, WIN, out=_bf16(1, 10, 4, 64), lse=lse)


@pytest.mark.parametrize("what", ["v", "k_batch", "head_dim", "out", "lse", "lse_dtype"])
def test_prefill_rejects_inconsistent_buffers(what):
    q, k, v = _bf16(1, 10, 4, 64), _bf16(1, 12, 2, 64), _bf16(1, 12, 2, 64)
    kw = {}
    win = WIN
    if what == "v":
        v = _bf16(1, 11, 2, 64)
    elif what == "k_batch":
        k, v = _bf16(2, 12, 2, 64), _bf16(2, 12, 2, 64)
    elif what == "head_dim":
        win = wp.Window(128, 1e4, 1.0, 1)
    elif what == "out":
        kw["out"] = _bf16(1, 10, 4, 32)
    elif what == "lse":
        kw["lse"] = torch.zeros((1, 4, 9), dtype=torch.float32)
    else:
        kw["lse"] = torch.zeros((1, 4, 10), dtype=torch.float64)
    with pytest.raises((ValueError, TypeError)) as e:
        wp.prefill(q, k, v, win, **kw)
    assert "CUDA" not in str(e.value)


def test_decode_consistent_shapes_reach_the_device_check():
    q, kc, vc = _bf16(2, 4, 64), _bf16(2, 50, 2, 64), _bf16(2, 50, 2, 64)
    with pytest.raises(TypeError, match="CUDA"):
        wp.decode(q, kc, vc, [50, 7], WIN, workspace=torch.zeros(1024, dtype=torch.uint8),
                  out=_bf16(2, 4, 64), lse=torch.zeros((2, 4), dtype=torch.float32))


@pytest.mark.parametrize("what", ["v_cache", "k_cache", "kv_len", "out", "lse", "head_dim"])
def test_decode_rejects_inconsistent_buffers(what):
    q, kc, vc = _bf16(2, 4, 64), _bf16(2, 50, 2, 64), _bf16(2, 50, 2, 64)
    kv_len = [50, 7]
    kw = {"workspace": torch.zeros(1024, dtype=torch.uint8)}
    win = WIN
    if what == "v_cache":
        vc = _bf16(2, 40, 2, 64)
    elif what == "k_cache":
        kc = _bf16(1, 50, 2, 64)
    elif what == "kv_len":
        kv_len = [50]
    elif what == "out":
        kw["out"] = _bf16(2, 2, 64)
    elif what == "lse":
        kw["lse"] = torch.zeros((2, 3), dtype=torch.float32)
    else:
        win = wp.Window(128, 1e4, 1.0, 1)
    with pytest.raises((ValueError, TypeError)) as e:
        wp.decode(q, kc, vc, kv_len, win, **kw)
    assert "CUDA" not in str(e.value)


@pytest.mark.parametrize("fn", ["prefill_masked", "prefill_rope", "prefill_positions"])
def test_prefill_variants_check_shapes_first(fn):
    q, k, v = _bf16(1, 10, 4, 64), _bf16(1, 12, 2, 64), _bf16(1, 11, 2, 64)   # v too short
    mask = torch.ones((1, 4, 1, 1), dtype=torch.bool)
    pos = torch.zeros((1, 16), dtype=torch.int32)
    args = {"prefill_masked": (q, k, v, mask, WIN), "prefill_rope": (q, k, v, WIN),
            "prefill_positions": (q, k, v, pos, pos, WIN)}[fn]
    with pytest.raises(ValueError, match="v has shape"):
        getattr(wp, fn)(*args)


def test_decode_variant_outputs_are_checked():
    q, kc, vc = _bf16(2, 4, 64), _bf16(2, 50, 2, 64), _bf16(2, 50, 2, 64)
    with pytest.raises(ValueError, match="lse has shape"):
        wp.decode_noalloc(q, kc, vc, [50, 7], WIN, lse=torch.zeros((2, 5), dtype=torch.float32))
