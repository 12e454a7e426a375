"""GPU asymmetric (zero-point) path against the oracle.

Codes, scales and zero points must equal the oracle's bit for bit; Y must
satisfy |Y - Y_ref| <= 2^-9 |Y_ref| + 1e-3 rms(Y_ref) element-wise against
the oracle's fp64 (q - z) S product.  Both linear kernels (weight streaming
for M <= 64, tensor cores above, with and without the K split) are covered.
"""
import numpy as np
import pytest

import oracle
import synthetic
from tests.gpu_helpers import SEED, assert_close, par_linear, par_quantize, to_gpu, to_np, w8

pytestmark = pytest.mark.gpu


def _asym_pipeline(W, X, bias=None):
    m = w8()
    q, s, z = m.quantize_asym(to_gpu(W))
    packed = m.prepack(q)
    Y = m.linear_asym(to_gpu(X), packed, s, z, None if bias is None else to_gpu(bias))
    return to_np(q), to_np(s), to_np(z), to_np(Y)


def _weights(K, N, tid, outliers=0.001):
    W = synthetic.weights(K, N, SEED, tid, outlier_frac=outliers)
    # sign-definite and all-zero channels: zero points at both ends and 0
    if N >= 32:
        W[:, 1] = np.abs(W[:, 1])
        W[:, 2] = -np.abs(W[:, 2])
        W[:, 3] = 0.0
        W[:, 4] = np.abs(W[:, 4]) + 0.05
    return W


@pytest.mark.parametrize("K,N", [(64, 8), (256, 512), (1000, 264), (4096, 4608), (6000, 264), (13696, 256),
                                 (300, 27392), (20000, 40)])
@pytest.mark.parametrize("dtype", [np.float32, np.float16])
def test_quantize_asym_bit_exact(K, N, dtype):
    m = w8()
    W = _weights(K, N, 5000 + K + N).astype(dtype)
    q, s, z = m.quantize_asym(to_gpu(W))
    qo, so, zo = oracle.quantize_asym(W)
    assert np.array_equal(to_np(q), qo)
    assert np.array_equal(to_np(s).view(np.uint16), so.view(np.uint16))
    assert np.array_equal(to_np(z), zo)


def test_quantize_asym_near_rounding_boundaries():
    # weights placed on and next to the half-integer boundaries of w / S
    m = w8()
    rng = np.random.default_rng(17)
    K, N = 2048, 64
    S = np.float32(2.0 ** -7)
    base = rng.integers(-120, 120, size=(K, N)).astype(np.float32) + 0.5
    W = (base * S).astype(np.float32)
    W = np.nextafter(W, np.where(rng.random((K, N)) < 0.5, np.float32(-np.inf), np.float32(np.inf)))
    W[: K // 3] = (base[: K // 3] * S).astype(np.float32)
    q, s, z = m.quantize_asym(to_gpu(W))
    qo, so, zo = oracle.quantize_asym(W)
    assert np.array_equal(to_np(q), qo) and np.array_equal(to_np(z), zo)
    assert np.array_equal(to_np(s).view(np.uint16), so.view(np.uint16))


def _check_asym(M, K, N, tid, bias=True):
    W = _weights(K, N, tid)
    X = synthetic.activations(M, K, SEED, tid + 1)
    b = synthetic.bias(N, SEED, tid + 2) if bias else None
    qg, sg, zg, Yg = _asym_pipeline(W, X, b)
    qo, so, zo = oracle.quantize_asym(W)
    assert np.array_equal(qg, qo) and np.array_equal(zg, zo)
    assert np.array_equal(sg.view(np.uint16), so.view(np.uint16))
    assert_close(Yg, oracle.linear_asym(X, qo, so, zo, b), f"asym M={M} K={K} N={N}")


@pytest.mark.parametrize("M", [1, 3, 16, 33, 64])
@pytest.mark.parametrize("K,N", [(256, 512), (1000, 264), (4096, 384)])
def test_linear_asym_decode(M, K, N):
    _check_asym(M, K, N, 5100 + M + K + N, bias=(M % 2 == 1))


@pytest.mark.parametrize("M", [65, 129, 300])
@pytest.mark.parametrize("K,N", [(256, 512), (520, 264), (4096, 384)])
def test_linear_asym_prefill(M, K, N):
    _check_asym(M, K, N, 5200 + M + K + N)


def test_linear_asym_prefill_k_split():
    # 2 pair tiles of 32 K steps: the K split over all pairs
    _check_asym(129, 8192, 512, 5300)


def test_linear_asym_exact_integers_bit_exact():
    # integer activations and weights on an exact grid: every product and
    # partial sum is an integer below 2^24, so Y is exact on both kernels
    m = w8()
    rng = np.random.default_rng(23)
    K, N = 512, 136
    S = np.float16(0.25)
    Z = rng.integers(-100, 100, N)
    I = rng.integers(-128, 128, size=(K, N))
    I[0], I[1] = -128, 127
    W = ((I - Z) * np.float32(S)).astype(np.float32)
    for M in (5, 100):
        X = rng.integers(-3, 4, size=(M, K)).astype(np.float16)
        qg, sg, zg, Yg = _asym_pipeline(W, X)
        qo, so, zo = oracle.quantize_asym(W)
        assert np.array_equal(qg, qo) and np.array_equal(zg, zo) and np.array_equal(zg.astype(np.int64), Z)
        Yref = oracle.linear_asym(X, qo, so, zo)
        assert np.array_equal(Yg.view(np.uint16), Yref.astype(np.float16).view(np.uint16)), M


def test_linear_asym_chatglm2_h_to_4h_decode_full():
    # every code, scale, zero point and output of the headline shape
    K, N = 4096, 27392
    tid = 5400
    W = _weights(K, N, tid)
    X = synthetic.activations(1, K, SEED, tid + 1)
    qg, sg, zg, Yg = _asym_pipeline(W, X)
    qo, so, zo = par_quantize(W, fn=oracle.quantize_asym)
    assert np.array_equal(sg.view(np.uint16), so.view(np.uint16))
    assert np.array_equal(qg, qo) and np.array_equal(zg, zo)
    assert_close(Yg, par_linear(X, qo, so, zo, fn=oracle.linear_asym), "asym h-to-4h decode")


def test_linear_asym_rejects_missing_zeros():
    torch = pytest.importorskip("torch")
    m = w8()
    lib = m.load_library()
    X = torch.zeros((4, 64), dtype=torch.float16, device="cuda")
    q, s, z = m.quantize_asym(torch.zeros((64, 128), dtype=torch.float32, device="cuda"))
    packed = m.prepack(q)
    Y = torch.empty((4, 128), dtype=torch.float16, device="cuda")
    ws = torch.zeros(m.workspace_bytes(4, 64, 128), dtype=torch.uint8, device="cuda")
    rc = lib.w8a16_linear_asym(X.data_ptr(), packed.data_ptr(), s.data_ptr(), None, None, Y.data_ptr(),
                               4, 64, 128, ws.data_ptr(), ws.numel(), None)
    assert rc == -1
    rc = lib.w8_quantize_per_channel_asym(X.data_ptr(), 0, 64, 128, q.data_ptr(), s.data_ptr(), None, None)
    assert rc == -1
