"""GPU clipped-scale quantization (fixed range and percentile) against the
oracle: codes and scales bit for bit, and the linear on clipped codes."""
import numpy as np
import pytest

import oracle
import synthetic
from tests.gpu_helpers import SEED, assert_close, to_gpu, to_np, w8

pytestmark = pytest.mark.gpu

SHAPES = [(64, 8), (256, 512), (1000, 264), (1024, 40), (1025, 40), (4096, 4608), (13696, 128)]


def _check(W, mode, param):
    m = w8()
    q, s = m.quantize_clip(to_gpu(W), mode, param)
    qo, so = oracle.quantize_clip(W, mode, param)
    assert np.array_equal(to_np(s).view(np.uint16), so.view(np.uint16)), (mode, param)
    assert np.array_equal(to_np(q), qo), (mode, param)


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("dtype", [np.float32, np.float16])
def test_percentile_clip_bit_exact(K, N, dtype):
    W = synthetic.weights(K, N, SEED, 6000 + K + N, outlier_frac=0.001).astype(dtype)
    for p in (0.999, 0.99, 0.5, 1.0, 1e-4):
        _check(W, "percentile", p)


@pytest.mark.parametrize("K,N", SHAPES)
def test_fixed_clip_bit_exact(K, N):
    W = synthetic.weights(K, N, SEED, 6100 + K + N, outlier_frac=0.001)
    for c in (0.03, 0.0, 1e30, float("inf"), 0.045):
        _check(W, "fixed", c)


def test_percentile_with_ties_and_zero_columns():
    # magnitudes on a coarse grid: many equal values around every rank
    rng = np.random.default_rng(31)
    K, N = 3000, 96
    W = (rng.integers(-20, 21, size=(K, N)) * 0.125).astype(np.float32)
    W[:, 7] = 0.0
    W[:, 8] = 0.5
    for p in (0.9, 0.5, 0.99, 1.0):
        _check(W, "percentile", p)


def test_percentile_crowded_leading_digits():
    # Half of each column's rows share their leading bits in large numbers:
    # 3000 values 0.5 (1 + m 2^-23) with m below 2^21, 2^10 or 2^3 carry one
    # leading 10-bit digit (more than a column can collect at once), and
    # with the smaller ranges also one or two further 7-bit digits, so the
    # selection goes on histogramming before it collects, or never collects.
    rng = np.random.default_rng(37)
    K, N = 6000, 72
    W = rng.normal(0.0, 0.02, size=(K, N)).astype(np.float32)
    for lo, hi, bits in ((0, 16, 21), (16, 32, 10), (48, 72, 3)):
        rows = rng.permutation(K)[:3000]
        m = rng.integers(0, 1 << bits, size=(3000, hi - lo))
        sign = np.where(rng.random((3000, hi - lo)) < 0.5, -1.0, 1.0)
        W[rows, lo:hi] = (sign * 0.5 * (1.0 + m * 2.0 ** -23)).astype(np.float32)
    for p in (0.9, 0.5, 0.25, 0.999, 1e-4):
        _check(W, "percentile", p)
    _check(W.astype(np.float16), "percentile", 0.5)


def test_percentile_matches_plain_quantizer_at_p_one():
    m = w8()
    W = synthetic.weights(2048, 1032, SEED, 6200, outlier_frac=0.01)
    q1, s1 = m.quantize(to_gpu(W))
    q2, s2 = m.quantize_clip(to_gpu(W), "percentile", 1.0)
    assert np.array_equal(to_np(q1), to_np(q2)) and np.array_equal(to_np(s1), to_np(s2))


def test_linear_on_clipped_codes():
    m = w8()
    K, N = 4096, 1024
    W = synthetic.weights(K, N, SEED, 6300, outlier_frac=0.001)
    for M in (1, 40, 200):
        X = synthetic.activations(M, K, SEED, 6301 + M)
        q, s = m.quantize_clip(to_gpu(W), "percentile", 0.999)
        Y = to_np(m.linear(to_gpu(X), m.prepack(q), s))
        qo, so = oracle.quantize_clip(W, "percentile", 0.999)
        assert np.array_equal(to_np(q), qo)
        assert_close(Y, oracle.linear(X, qo, so), f"clipped M={M}")


def test_clip_rejects_bad_arguments():
    torch = pytest.importorskip("torch")
    m = w8()
    lib = m.load_library()
    W = torch.zeros((64, 8), dtype=torch.float32, device="cuda")
    q = torch.empty((64, 8), dtype=torch.int8, device="cuda")
    s = torch.empty((8,), dtype=torch.float16, device="cuda")
    call = lambda mode, prm: lib.w8_quantize_per_channel_clip(W.data_ptr(), 0, 64, 8, mode, prm, q.data_ptr(),
                                                              s.data_ptr(), None)
    assert call(1, 0.0) == -2 and call(1, 1.5) == -2 and call(1, float("nan")) == -2
    assert call(0, -1.0) == -2 and call(0, float("nan")) == -2
    assert call(7, 0.5) == -4
    assert call(1, 0.5) == 0 and call(0, 0.5) == 0
