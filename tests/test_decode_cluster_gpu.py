"""The decode kernel's cluster form: few channel blocks, up to 16 tokens.

A thread-block cluster of C CTAs owns one 128-channel block and splits its
K range evenly; CTA 0 adds the others' fp32 parts (stored into its shared
memory) in rank order.  The host takes this form when the blocks alone
would leave SMs idle: C is the largest cluster size that keeps one cluster
per block resident at once and at least one K block per CTA.  These cases
span C = 2 .. 8 (the number of channel blocks sets C), ragged K (shares of
unequal length) and ragged N, every token count of the form, with and
without bias, both code forms and the outlier split; every output is
checked against the oracle, and repeated calls must give the same bits.
"""
import numpy as np
import pytest

import oracle
import synthetic
from tests.gpu_helpers import SEED, assert_close, par_linear, par_quantize, to_gpu, to_np, w8

pytestmark = pytest.mark.gpu

# (K, N): N / 128 channel blocks of 18 .. 74 -> cluster sizes 8 .. 2 on 148
# SMs; K from 1000 (16 K blocks, uneven shares) to 13696
SHAPES = [(4096, 2304), (1000, 2560), (4096, 3200), (13696, 4096), (4096, 4608), (2048, 6144),
          (512, 9472), (4096, 4096)]


def _case(M, K, N, tid, bias):
    W = synthetic.weights(K, N, SEED, tid, outlier_frac=0.001)
    X = synthetic.activations(M, K, SEED, tid + 1)
    b = synthetic.bias(N, SEED, tid + 2) if bias else None
    return W, X, b


@pytest.mark.parametrize("K,N", SHAPES)
def test_cluster_decode_matches_oracle(K, N):
    m = w8()
    tid = 12000 + K + N
    W, _, _ = _case(1, K, N, tid, False)
    q, s = m.quantize(to_gpu(W))
    packed = m.prepack(q)
    qo, so = par_quantize(W)
    assert np.array_equal(to_np(q), qo)
    for M in (1, 2, 7, 8, 9, 15, 16):
        _, X, b = _case(M, K, N, tid + 10 * M, bias=(M % 2 == 1))
        Xg, bg = to_gpu(X), (None if b is None else to_gpu(b))
        Y = to_np(m.linear(Xg, packed, s, bg))
        assert_close(Y, par_linear(X, qo, so, bias=b), f"M={M} K={K} N={N}")
        Y2 = to_np(m.linear(Xg, packed, s, bg))
        assert np.array_equal(Y.view(np.uint16), Y2.view(np.uint16)), "not repeatable"


def test_cluster_decode_exact_integers_bit_exact():
    # integer activations and power-of-two-multiple weights: every partial
    # sum is exact in fp32, so the rank-order sum must give the exact value
    rng = np.random.default_rng(5)
    K, N = 2048, 4096
    for M in (1, 16):
        X = rng.integers(-8, 9, size=(M, K)).astype(np.float16)
        s0 = 2.0 ** rng.integers(-10, -4, size=N)
        j = rng.integers(-127, 128, size=(K, N))
        j[0] = 127
        W = (j * s0).astype(np.float32)
        m = w8()
        q, s = m.quantize(to_gpu(W))
        Y = to_np(m.linear(to_gpu(X), m.prepack(q), s))
        qo, so = oracle.quantize(W)
        Yref = oracle.linear(X, qo, so)
        assert np.array_equal(Y.view(np.uint16), Yref.astype(np.float16).view(np.uint16))


@pytest.mark.parametrize("M", [1, 16])
def test_cluster_decode_asymmetric_codes(M):
    m = w8()
    K, N = 4096, 4096
    W = synthetic.weights(K, N, SEED, 12500, outlier_frac=0.001)
    X = synthetic.activations(M, K, SEED, 12501 + M)
    q, s, z = m.quantize_asym(to_gpu(W))
    Y = to_np(m.linear_asym(to_gpu(X), m.prepack(q), s, z))
    qo, so, zo = par_quantize(W, fn=oracle.quantize_asym)
    assert np.array_equal(to_np(q), qo) and np.array_equal(to_np(z), zo)
    assert_close(Y, par_linear(X, qo, so, zo, fn=oracle.linear_asym), f"asym M={M}")


@pytest.mark.parametrize("M", [1, 16])
def test_cluster_decode_outlier_split(M):
    m = w8()
    K, N = 4096, 4608
    W = synthetic.weights(K, N, SEED, 12600, outlier_frac=0.001)
    X = synthetic.activations(M, K, SEED, 12601 + M)
    q, s, c, r, v = m.quantize_outliers(to_gpu(W), 0.999)
    Y = to_np(m.linear_outliers(to_gpu(X), m.prepack(q), s, c, r, v))
    o = par_quantize(W, fn=lambda w: oracle.quantize_outliers(w, 0.999))
    assert_close(Y, par_linear(X, *o, fn=oracle.linear_outliers), f"outliers M={M}")


def test_cluster_decode_leaves_workspace_counters_alone():
    # the cluster form uses no workspace: a zeroed workspace stays zero,
    # and the stream-K form that follows on it is still right
    torch = pytest.importorskip("torch")
    m = w8()
    K, N = 4096, 4096
    W, X, _ = _case(1, K, N, 12700, False)
    q, s = m.quantize(to_gpu(W))
    packed = m.prepack(q)
    ws = torch.zeros(m.workspace_bytes(1, K, N), dtype=torch.uint8, device="cuda")
    m.linear(to_gpu(X), packed, s, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws.count_nonzero()) == 0
    W2, X2, _ = _case(1, 4096, 27392, 12710, False)
    q2, s2 = m.quantize(to_gpu(W2))
    Y2 = to_np(m.linear(to_gpu(X2), m.prepack(q2), s2, workspace=ws))
    qo, so = par_quantize(W2)
    assert_close(Y2, par_linear(X2, qo, so), "stream-K after the cluster form")
    assert m.device_status() == 0
