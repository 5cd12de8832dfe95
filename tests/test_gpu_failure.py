"""Failure detection on the GPU without a GPU fault.

Every pipeline wait in the kernels is bounded; when one gives up the kernel sets
a bit in the per-device error word and returns normally.  The self-test entry
point runs that same bounded wait on a barrier nothing completes, so the wait
really runs out; the host then reads the status, and the device must still work.
"""
import time

import numpy as np
import pytest
import torch

from test_gpu_parity import _fixed, _run_and_compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from paged_kv_cache_393_b200 import build
    build.build()
    import paged_kv_cache_393_b200 as m
    m.device_errors(clear=True)
    return m


def test_a_wait_that_runs_out_is_reported_and_the_device_stays_usable(pkv):
    t0 = time.perf_counter()
    pkv.selftest_wait_timeout(20_000)              # 20 ms
    flags = pkv.device_errors(clear=True)          # synchronizes
    elapsed = time.perf_counter() - t0
    assert flags == pkv.DEVERR_TIMEOUT
    assert elapsed >= 0.02
    assert pkv.device_errors(clear=True) == 0      # cleared
    # the context is intact: both attention kernels still match the oracle
    _run_and_compare(pkv, _fixed("after_timeout_mha", 8, 8, 128, 16, [5, 300]))
    _run_and_compare(pkv, _fixed("after_timeout_gqa", 16, 2, 128, 16, [5, 900]), partition_size=256)


def test_self_test_rejects_bad_timeouts(pkv):
    from paged_kv_cache_393_b200 import PagedKVError
    with pytest.raises(PagedKVError):
        pkv.selftest_wait_timeout(0)
    with pytest.raises(PagedKVError):
        pkv.selftest_wait_timeout(2_000_000)
