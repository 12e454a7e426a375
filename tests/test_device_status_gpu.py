"""Bounded device waits: a wait that nothing completes gives up after its
limit, records its site in the status word and the kernel returns; the
context stays usable afterwards."""
import pytest

from tests.gpu_helpers import w8

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_reports_and_returns():
    m = w8()
    assert m.device_status() == 0
    m.test_bounded_wait(2_000_000)          # 2 ms limit
    st = m.device_status()
    assert st & 1 and (st >> 8) & 0xFF == 0xEE
    assert m.device_status() == 0           # read-and-clear


def test_normal_calls_leave_status_clear():
    import numpy as np
    from tests.gpu_helpers import gpu_pipeline
    import synthetic
    W = synthetic.weights(256, 512, 1, 1)
    for M in (1, 16, 64):
        X = synthetic.activations(M, 256, 1, 2)
        gpu_pipeline(W, X)
    assert m_status() == 0


def m_status():
    return w8().device_status()
