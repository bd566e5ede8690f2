"""Failure detection without a fault: every wait in the library is bounded,
and a wait that runs out records FA_ERR_TIMEOUT and its site, raises the
CTA's abort flag so that the CTA's other waiting warps leave at once, and
returns; the context stays usable.  fa_selftest_wait_timeout runs that path
on purpose, with the library's own wait, on an mbarrier phase that nothing
completes (no bad address, no trap, no unbounded loop).
"""
import time

import pytest
import torch

import flash_fwd_b200 as fa
from flash_fwd_b200 import inputs

FA_ERR_INVALID_ARG = 1
FA_ERR_TIMEOUT = 6
BOUND_S = 3.0           # the library's bound per wait
STAGGER_S = 0.1         # warp w starts its wait w x 100 ms after the CTA starts


@pytest.mark.parametrize("warps", [0, 33, -1])
def test_selftest_refuses_bad_warp_counts_before_launching(warps):
    rc, site = fa.fa_selftest_wait_timeout(warps)
    assert rc == FA_ERR_INVALID_ARG and site == (0, 0, 0, 0, 0)


@pytest.mark.gpu
def test_single_wait_runs_out_and_reports_its_site():
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    rc, site = fa.fa_selftest_wait_timeout(1)
    dt = time.perf_counter() - t0
    assert rc == FA_ERR_TIMEOUT, fa.fa_status_string(rc)
    bx, by, warp, bar_addr, parity = site
    assert (bx, by, warp, parity) == (0, 0, 0, 0)
    assert bar_addr % 8 == 0          # a shared-memory mbarrier address
    assert BOUND_S * 0.95 <= dt <= BOUND_S + 2.0


@pytest.mark.gpu
def test_abort_flag_releases_the_other_warps():
    # without the abort flag the last warp would give up at 3 s + 31 x 100 ms
    # = 6.1 s.  Which warp notices its bound first is not fixed: a wait
    # checks the clock every 32 try_wait calls, and each may suspend the warp
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    rc, site = fa.fa_selftest_wait_timeout(32)
    dt = time.perf_counter() - t0
    assert rc == FA_ERR_TIMEOUT
    assert site[:2] == (0, 0) and 0 <= site[2] < 32 and site[4] == 0
    assert BOUND_S * 0.95 <= dt < BOUND_S + 31 * STAGGER_S * 0.5


@pytest.mark.gpu
def test_context_stays_usable_and_the_library_word_is_untouched():
    fa.fa_selftest_wait_timeout(4)
    # the attention kernels' status word saw nothing
    assert fa.fa_last_device_status() == 0
    from parity import check_fwd, gpu_fwd
    q, k, v, _ = inputs.make_qkv(1, 2, 300, 128, "bf16", seed=5, with_dout=False)
    scale = inputs.default_scale(128)
    o, lse = gpu_fwd(q, k, v, True, scale)
    check_fwd(o, lse, q, k, v, True, scale, "bf16")
