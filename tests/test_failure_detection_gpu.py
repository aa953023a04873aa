"""The library's bounded-wait failure path on the GPU, without a fault.

Every wait in the library's kernels (mbarrier phases of the TMA rings, the
tensor-core hand-offs) is bounded on the device's global timer; when a bound
runs out the waiting thread records WPATTN_ETIMEOUT in the device status word
and the kernel returns.  The self-check kernel waits on a barrier that nothing
ever arrives at, so its bound must run out: the status must then read
WPATTN_ETIMEOUT exactly once, and the context must stay usable for a normal
call afterwards.
"""
import math
import time

import numpy as np
import pytest
import torch

import oracle
import rope_wavelength_sparsity_b200 as wp
from rope_wavelength_sparsity_b200 import inputs

pytestmark = pytest.mark.gpu


def test_wait_bound_runs_out_and_is_reported(cuda_dev):
    wp.device_status()                              # start from a cleared status word
    t0 = time.perf_counter()
    wp.selftest_wait_timeout()
    status = wp.device_status()                     # synchronises, reads and clears
    elapsed = time.perf_counter() - t0
    assert status == wp.ETIMEOUT
    assert 1.5 < elapsed < 30.0                     # the 2 s bound ran out, then the kernel returned
    assert wp.device_status() == wp.OK              # cleared by the read


def test_context_usable_after_a_timeout(cuda_dev):
    wp.selftest_wait_timeout()
    assert wp.device_status() == wp.ETIMEOUT
    B, Hq, Hkv, D, L = 1, 4, 2, 64, 300
    q = inputs.randn_bf16((B, Hq, D), 11)
    kc = inputs.randn_bf16((B, L, Hkv, D), 12)
    vc = inputs.randn_bf16((B, L, Hkv, D), 13)
    win = wp.Window(D, 1e4, 1.0, 1)
    out, lse = wp.decode(q.cuda(), kc.cuda(), vc.cuda(), [L], win)
    assert wp.device_status() == wp.OK
    o_ref, l_ref = oracle.decode_rows(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), [L],
                                      Hq=Hq, Hkv=Hkv, base=1e4, alpha=1.0, g=1,
                                      scale=1 / math.sqrt(D))
    oc = out.float().cpu().reshape(B * Hq, D).numpy()
    lc = lse.cpu().reshape(-1).numpy()
    assert np.abs(oc - o_ref).max() <= 1e-2
    assert np.abs(lc - l_ref).max() <= 2e-3


def test_check_option_raises_on_a_timeout(cuda_dev):
    """``check=True`` synchronises and turns a nonzero status word into an error; a
    clean call with it returns normally."""
    B, Hq, Hkv, D, L = 1, 4, 2, 64, 300
    q = inputs.randn_bf16((B, Hq, D), 21).cuda()
    kc = inputs.randn_bf16((B, L, Hkv, D), 22).cuda()
    vc = inputs.randn_bf16((B, L, Hkv, D), 23).cuda()
    win = wp.Window(D, 1e4, 1.0, 1)
    wp.device_status()
    wp.decode(q, kc, vc, [L], win, check=True)       # clean: no error
    wp.selftest_wait_timeout()                        # the status word now holds ETIMEOUT
    with pytest.raises(wp.WpattnError) as err:
        wp.decode(q, kc, vc, [L], win, check=True)
    assert err.value.code == wp.ETIMEOUT
    assert wp.device_status() == wp.OK                # the check's read cleared it
