"""GPU outlier split against the oracle: codes, scales and the fp16 side
list bit for bit; Y within tolerance on both linear kernels."""
import numpy as np
import pytest

import oracle
import synthetic
from tests.gpu_helpers import SEED, assert_close, par_linear, par_quantize, to_gpu, to_np, w8

pytestmark = pytest.mark.gpu


def _split(W, p):
    m = w8()
    q, s, c, r, v = m.quantize_outliers(to_gpu(W), p)
    return tuple(to_np(t) for t in (q, s, c, r, v))


@pytest.mark.parametrize("K,N", [(64, 8), (1000, 264), (4096, 4608), (13696, 128)])
@pytest.mark.parametrize("dtype", [np.float32, np.float16])
def test_quantize_outliers_bit_exact(K, N, dtype):
    W = synthetic.weights(K, N, SEED, 7000 + K + N, outlier_frac=0.001).astype(dtype)
    for p in (0.999, 0.99, 1.0):
        if K - int(np.ceil(p * K)) > 64:
            continue
        g = _split(W, p)
        o = oracle.quantize_outliers(W, p)
        assert np.array_equal(g[0], o[0]), p
        assert np.array_equal(g[1].view(np.uint16), o[1].view(np.uint16)), p
        assert np.array_equal(g[2], o[2]) and np.array_equal(g[3], o[3]), p
        assert np.array_equal(g[4].view(np.uint16), o[4].view(np.uint16)), p


def _check(M, K, N, p, tid, bias=True):
    m = w8()
    W = synthetic.weights(K, N, SEED, tid, outlier_frac=0.002)
    X = synthetic.activations(M, K, SEED, tid + 1)
    b = synthetic.bias(N, SEED, tid + 2) if bias else None
    q, s, c, r, v = m.quantize_outliers(to_gpu(W), p)
    Y = to_np(m.linear_outliers(to_gpu(X), m.prepack(q), s, c, r, v, None if b is None else to_gpu(b)))
    o = oracle.quantize_outliers(W, p)
    assert np.array_equal(to_np(q), o[0]) and np.array_equal(to_np(r), o[3])
    assert_close(Y, oracle.linear_outliers(X, *o, bias=b), f"outliers M={M} K={K} N={N}")


@pytest.mark.parametrize("M", [1, 7, 33, 64, 65, 300, 600])
@pytest.mark.parametrize("K,N", [(520, 264), (4096, 384), (1000, 1032)])
def test_linear_outliers(M, K, N):
    _check(M, K, N, 0.995, 7100 + M + K + N, bias=(M % 2 == 1))


def test_linear_outliers_chatglm2_h_to_4h_full():
    # every code, scale, side-list entry and output of the headline shape,
    # through the weight-streaming (M = 1) and tensor-core (M = 256) paths
    m = w8()
    K, N = 4096, 27392
    W = synthetic.weights(K, N, SEED, 7200, outlier_frac=0.001)
    q, s, c, r, v = m.quantize_outliers(to_gpu(W), 0.999)
    o = par_quantize(W, fn=lambda w: oracle.quantize_outliers(w, 0.999))
    assert np.array_equal(to_np(q), o[0]) and np.array_equal(to_np(s).view(np.uint16), o[1].view(np.uint16))
    assert np.array_equal(to_np(c), o[2]) and np.array_equal(to_np(r), o[3])
    assert np.array_equal(to_np(v).view(np.uint16), o[4].view(np.uint16))
    packed = m.prepack(q)
    for M in (1, 256):
        X = synthetic.activations(M, K, SEED, 7201 + M)
        Y = to_np(m.linear_outliers(to_gpu(X), packed, s, c, r, v))
        assert_close(Y, par_linear(X, *o, fn=oracle.linear_outliers), f"h-to-4h outliers M={M}")


def test_outlier_capacity_limit():
    torch = pytest.importorskip("torch")
    m = w8()
    lib = m.load_library()
    assert lib.w8_outlier_capacity(4096, 0.999) == 4 and lib.w8_outlier_capacity(4096, 1.0) == 0
    W = torch.zeros((4096, 8), dtype=torch.float32, device="cuda")
    q = torch.empty((4096, 8), dtype=torch.int8, device="cuda")
    s = torch.empty((8,), dtype=torch.float16, device="cuda")
    c = torch.empty((8,), dtype=torch.int32, device="cuda")
    r = torch.empty((8, 100), dtype=torch.int32, device="cuda")
    v = torch.empty((8, 100), dtype=torch.float16, device="cuda")
    rc = lib.w8_quantize_per_channel_outliers(W.data_ptr(), 0, 4096, 8, 0.98, q.data_ptr(), s.data_ptr(),
                                              c.data_ptr(), r.data_ptr(), v.data_ptr(), None)
    assert rc == -10
