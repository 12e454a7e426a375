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


def test_wait_that_runs_out_resets_default_workspaces():
    # A kernel whose wait gave up may leave split-K counters set in the
    # workspace it used.  Reading the status resets the binding's default
    # workspaces, so the next call without workspace= starts clean.  The
    # stale counters are planted by hand (every byte of the default
    # workspace set to 1) before a wait is made to run out.
    import numpy as np
    import oracle
    import synthetic
    from tests.gpu_helpers import assert_close, to_gpu, to_np
    m = w8()
    K, N = 4096, 4096
    W = synthetic.weights(K, N, 1, 3)
    X = synthetic.activations(1, K, 1, 4)
    q, s = m.quantize(to_gpu(W))
    packed = m.prepack(q)
    Xg = to_gpu(X)
    m.linear(Xg, packed, s)                  # creates this stream's default workspace
    assert m.device_status() == 0
    import torch
    key = (0, torch.cuda.current_stream(0).cuda_stream)
    ws = m._ws_cache[key]
    ws.fill_(1)
    m.test_bounded_wait(2_000_000)
    assert m.device_status() != 0            # the wait ran out ...
    assert int(ws.count_nonzero()) == 0      # ... and the default workspace was zeroed
    qo, so = oracle.quantize(W)
    assert_close(to_np(m.linear(Xg, packed, s)), oracle.linear(X, qo, so), "after reset")
    assert m.device_status() == 0
