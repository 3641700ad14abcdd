"""A device wait that runs out: the self-test kernel waits on a barrier that nothing completes;
its bounded wait gives up after the library's limit (2 s) and records QT2_ERR_TIMEOUT, which
qt2_device_status reports once and clears.  The context then still computes correct results.
(Runs last: it takes the full wait limit.)"""
import pytest
import torch

import oracle as O
from nvfp4_quantized_b200 import qt2
from tests.test_gpu_quant import _assert_view_equal, _inputs, gpu_fwd46

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert qt2.qt2_device_status() == 0
    qt2.qt2_selftest_wait_timeout()
    assert qt2.qt2_device_status() == qt2.QT2_ERR_TIMEOUT
    assert qt2.qt2_device_status() == 0          # read once, then cleared
    x = _inputs("gauss", 256, 384, seed=3)
    _assert_view_equal(gpu_fwd46(x), O.fwd46(x), "after the timeout")
    assert qt2.qt2_device_status() == 0
