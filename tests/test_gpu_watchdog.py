"""Failure detection on the device without a fault: the bounded waits that
every GEMM pipeline role uses give up, record QOQ_ERR_TIMEOUT with their wait
site, and return; the context stays usable afterwards."""
import numpy as np
import pytest

import oracle
from w4a8_quantized_gemm_qoq_b200 import inputs, qoq
from gpu_helpers import check_full, torch

pytestmark = [pytest.mark.gpu]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch().cuda.is_available(), "GPU tests need a CUDA device"
    from w4a8_quantized_gemm_qoq_b200 import build
    build.build()
    yield


def test_bounded_waits_time_out_and_report():
    t0 = torch().cuda.Event(enable_timing=True)
    t1 = torch().cuda.Event(enable_timing=True)
    t0.record()
    st = qoq.watchdog_selftest(limit_ns=50_000_000)
    t1.record()
    torch().cuda.synchronize()
    assert st[0:4] == [qoq.QOQ_ERR_TIMEOUT, 4, 0, 1], st[0:4]     # mbarrier phase that never completes
    assert st[8:12] == [qoq.QOQ_ERR_TIMEOUT, 6, 0, 2], st[8:12]   # flag that nothing sets
    assert st[16] == 0
    ms = t0.elapsed_time(t1)
    assert 45.0 <= ms < 1000.0, ms                                # gave up after about the limit


def test_context_usable_after_timeouts():
    qoq.watchdog_selftest(limit_ns=20_000_000)
    X = inputs.make_activations(16, 512, seed=5)
    W = inputs.make_weights(256, 512, seed=5)
    check_full(X, W, 128, "after watchdog self-test")
