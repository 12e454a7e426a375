"""The allocation-free decode entry point, w8a16_linear_decode_static.

Some callers cannot allocate device memory: an operator plugged into a host
framework whose fixed signature has no workspace argument, or a serving loop
whose memory is planned up front by another allocator and where a cudaMalloc
would synchronize the device.  For them the library keeps the decode
kernel's split-K scratch in a fixed array of static device memory.  This
test calls that entry point through the C ABI and checks it against the
regular entry point (w8a16_linear with a caller workspace) on two calls in
a row, so the second call runs on whatever the first left in the shared
array.  Both run the same decode kernel with the same split of the weight
over the SMs and add the split-K parts in the same order, so their outputs
must agree bit for bit; one case is also checked against the oracle
directly, and the split-K paths that timing rarely takes are forced (the
test hook that delays a CTA's count) so they too run on the static array.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synthetic
from tests.gpu_helpers import SEED, to_gpu, to_np, w8

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _static_call(lib, X, packed, scales, bias, Y):
    import torch
    M, K = X.shape
    N = scales.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.w8a16_linear_decode_static(_ptr(X), _ptr(packed), _ptr(scales), _ptr(bias),
                                          _ptr(Y), M, K, N, stream)


# (M, K, N): split-K with a counter per channel block (4096 x 4608), a wide
# layer whose CTAs span three channel blocks (4096 x 27392), a tall one
# (13696 x 264) and ragged ones; M across both token tilings of the kernel.
CASES = [(1, 4096, 4608), (16, 4096, 27392), (5, 13696, 264), (9, 1000, 1032), (3, 200, 136)]


def _run_cases(m, lib):
    import torch
    for i, (M, K, N) in enumerate(CASES):
        tid = 9000 + 10 * i
        W = synthetic.weights(K, N, SEED, tid, outlier_frac=0.001)
        X = to_gpu(synthetic.activations(M, K, SEED, tid + 1))
        b = to_gpu(synthetic.bias(N, SEED, tid + 2)) if i % 2 == 0 else None
        q, s = m.quantize(to_gpu(W))
        packed = m.prepack(q)
        Y_ws = to_np(m.linear(X, packed, s, b))
        for call in range(2):
            Y = torch.full((M, N), float("nan"), dtype=torch.float16, device=X.device)
            rc = _static_call(lib, X, packed, s, b, Y)
            assert rc == 0, m.STATUS.get(rc, rc)
            bad = np.argwhere(to_np(Y).view(np.uint16) != Y_ws.view(np.uint16))
            assert bad.size == 0, f"M={M} K={K} N={N} call {call}: {len(bad)} outputs differ, first {tuple(bad[0])}"
        if i == 0:
            # the oracle's own codes and fp64 product, within the tolerance
            qo, so = oracle.quantize(W)
            assert np.array_equal(to_np(q), qo)
            ok, worst = oracle.tolerance_ok(to_np(Y).astype(np.float64),
                                            oracle.linear(to_np(X), qo, so, None if b is None else to_np(b)))
            assert ok, f"against the oracle: worst err/bound {worst:.3f}"


def test_static_scratch_decode_matches_workspace_decode():
    m = w8()
    lib = m.load_library()
    _run_cases(m, lib)
    assert m.device_status() == 0


def test_static_scratch_rare_split_paths():
    # the hook delays each CTA's count of the part it publishes mid-stream,
    # so the late-finish and general split-K paths run on the static array
    m = w8()
    lib = m.load_library()
    m.test_set_decode_helper_delay(200_000)
    try:
        _run_cases(m, lib)
    finally:
        m.test_set_decode_helper_delay(0)
    assert m.device_status() == 0
    _run_cases(m, lib)          # and the array is left fit for normal use
    assert m.device_status() == 0


def test_static_scratch_rejects_sizes_beyond_its_limit():
    import torch
    m = w8()
    lib = m.load_library()
    K, N = 256, 512
    q, s = m.quantize(to_gpu(synthetic.weights(K, N, SEED, 9100)))
    packed = m.prepack(q)
    X = to_gpu(synthetic.activations(17, K, SEED, 9101))
    Y = torch.empty((17, N), dtype=torch.float16, device=X.device)
    assert _static_call(lib, X, packed, s, None, Y) == -10          # M > 16
    big = (1 << 20) + 8
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.w8a16_linear_decode_static(_ptr(X), _ptr(packed), _ptr(s), None, _ptr(Y),
                                          1, K, big, stream) == -10  # N > 2^20
    assert lib.w8_error_string(-10).decode().startswith("size beyond the fixed scratch")
