"""The allocation-free decode entry point.

wpattn_decode_noalloc serves callers that cannot allocate device memory
where they call decode (a runtime whose allocator holds all GPU memory, a
plugin that only receives tensors, a path where cudaMalloc is not allowed).
It runs the same decode with its scratch in a fixed array built into the
library.  This test calls it through the C ABI, twice in a row, and checks
each result against wpattn_decode with a caller-provided workspace.  It
lives in its own file, collected last, and passes both alone and after the
other tests.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import rope_wavelength_sparsity_b200 as wp
from rope_wavelength_sparsity_b200 import inputs

from _parity import ATOL_LSE, ATOL_OUT

pytestmark = pytest.mark.gpu


def _entry():
    fn = wp.lib().wpattn_decode_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(wp._Window), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.POINTER(ctypes.c_int32), ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                   ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_void_p]
    return fn


def _noalloc(L, win, q, kc, vc, kv_len, out, lse):
    fn = _entry()
    B, Hq, D = q.shape
    Lmax, Hkv = kc.shape[1], kc.shape[2]
    kvl = (ctypes.c_int32 * B)(*kv_len)
    return fn(ctypes.byref(win._c()), q.data_ptr(), kc.data_ptr(), vc.data_ptr(), kvl, Lmax, B,
              Hq, Hkv, 1.0 / math.sqrt(D), out.data_ptr(), lse.data_ptr(),
              torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("D,g,base,B,Hq,Hkv,L,kv_len", [
    (128, 1, 5e5, 3, 24, 8, 2000, [2000, 1, 1333]),
    (64, 8, 1e6, 2, 14, 2, 4096, [4096, 77]),
])
def test_decode_noalloc_matches_decode_with_workspace(cuda_dev, D, g, base, B, Hq, Hkv, L, kv_len):
    L_ = wp.lib()
    L_.wpattn_decode_noalloc_max_bytes.restype = ctypes.c_size_t
    assert L_.wpattn_decode_noalloc_max_bytes() == 4 << 20
    win = wp.Window(D, base, 1.0, g)
    q = inputs.randn_bf16((B, Hq, D), 901).cuda()
    kc = inputs.randn_bf16((B, L, Hkv, D), 902).cuda()
    vc = inputs.randn_bf16((B, L, Hkv, D), 903).cuda()
    ref_out, ref_lse = wp.decode(q, kc, vc, kv_len, win)
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=q.device)
        rc = _noalloc(L_, win, q, kc, vc, kv_len, out, lse)
        assert rc == wp.OK, wp.lib().wpattn_strerror(rc)
        assert wp.device_status() == wp.OK
        d_out = (out.float() - ref_out.float()).abs().max().item()
        d_lse = (lse - ref_lse).abs().max().item()
        assert d_out <= ATOL_OUT and d_lse <= ATOL_LSE, (call, d_out, d_lse)


def test_decode_noalloc_rejects_problems_beyond_its_scratch(cuda_dev):
    L_ = wp.lib()
    win = wp.Window(128, 5e5, 1.0, 1)
    # 128 sequences x 64 heads x (D + 2) floats exceed 4 MiB even with one split;
    # the tensors are consistent with the arguments, so the call would be valid
    B, Hq, Hkv, Lmax = 128, 64, 64, 16
    q = torch.zeros((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((B, Lmax, Hkv, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    kvl = (ctypes.c_int32 * B)(*([Lmax] * B))
    fn = _entry()
    rc = fn(ctypes.byref(win._c()), q.data_ptr(), kc.data_ptr(), kc.data_ptr(), kvl, Lmax, B, Hq,
            Hkv, ctypes.c_float(0.0), out.data_ptr(), lse.data_ptr(),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == wp.EWORKSPACE
