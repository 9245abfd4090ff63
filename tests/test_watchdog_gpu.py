"""Failure detection on the GPU without a GPU fault.

Every wait in the kernels is bounded.  fa_selftest_watchdog runs the same
bounded-wait code on a barrier that nothing ever arrives on; the wait must
give up after its limit, the error must reach the host as
FA_ERR_DEVICE_TIMEOUT, and the context must stay usable for the next call.
"""
import time

import pytest
import torch

from exact_attention_117_b200 import fa
from exact_attention_117_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    fa.check_device_error()  # start clean
    t0 = time.perf_counter()
    fa.selftest_watchdog(200)
    with pytest.raises(fa.FaError) as ei:
        fa.check_device_error()
    waited = time.perf_counter() - t0
    assert ei.value.status == 8
    assert "0x8000" in str(ei.value)
    assert 0.15 < waited < 5.0
    fa.check_device_error()  # the word was cleared by the read
    # the context is still usable: a small forward runs and is finite
    w = Workload("after", 1, 1, 200, 64, seed_base=3)
    x = make_inputs(w, "cuda", with_do=False)
    o, lse = fa.forward(x["q"], x["k"], x["v"], causal=True)
    fa.check_device_error()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_selftest_rejects_bad_limits():
    assert fa.load().fa_selftest_watchdog(0, None) == 2
    assert fa.load().fa_selftest_watchdog(5000, None) == 2
