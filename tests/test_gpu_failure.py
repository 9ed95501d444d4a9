"""Failure detection without a GPU fault: the bounded on-chip waits.

The attention kernel's pipeline waits give up after a time limit, report
PKV_DEVERR_TIMEOUT in the device error word and make the CTA's other warps
stop waiting, so a protocol bug can never hang the GPU.  Here a diagnostic
kernel waits on barriers that nothing arrives on: the first wait runs out
after 20 ms, the second (with the kernel's 2 s limit) ends early through the
abort flag, the host reads the error status, and the context stays usable.
"""
import time

import pytest
import torch

import oracle
import paged_kv_cache_420_b200 as pkv
import workloads
from tests._gpu_util import assert_attention_close, run_step, to_cuda

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    pkv.get_device_error()
    t0 = time.perf_counter()
    res = pkv.selftest_bounded_wait(20_000_000)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    first_done, second_done, second_us = res.tolist()
    assert first_done == 0 and second_done == 0
    assert second_us < 1_000_000  # gave up through the abort flag, not its own 2 s limit
    assert elapsed < 1.5
    assert pkv.get_device_error() == pkv.DEVERR_TIMEOUT
    # the context is still usable: a decode step after the timeout is correct
    w = to_cuda(workloads.make("tiny", seed=3))
    _, _, out = run_step(w)
    assert pkv.get_device_error() == 0
    assert_attention_close(out, oracle.decode_step(w)[2], "after timeout")


def test_bounded_wait_rejects_bad_limits():
    with pytest.raises(pkv.PkvError):
        pkv.selftest_bounded_wait(0)
    with pytest.raises(pkv.PkvError):
        pkv.selftest_bounded_wait(5_000_000_000)
