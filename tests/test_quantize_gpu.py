"""GPU quantization is bit-exact with the oracle (q and scales), on ragged
shapes, both weight dtypes, the edge columns the method has, and every
cluster split of the K range the kernel takes (1 to 4 CTAs for K <= 8192,
8 above, rows per CTA ragged at the end)."""
import numpy as np
import pytest

import oracle
import synthetic
from tests.gpu_helpers import SEED, par_quantize, to_gpu, to_np, w8

pytestmark = pytest.mark.gpu

SHAPES = [(256, 512), (1, 8), (7, 24), (63, 136), (65, 264), (200, 40), (1000, 1032), (4096, 512),
          (4097, 72), (5000, 136), (8192, 264), (8193, 40), (16384, 64), (16392, 24)]


def _gpu_quant(W):
    q, s = w8().quantize(to_gpu(W))
    return to_np(q), to_np(s)


def _check(W):
    qo, so = oracle.quantize(W)
    qg, sg = _gpu_quant(W)
    assert np.array_equal(sg.view(np.uint16), so.view(np.uint16))
    assert np.array_equal(qg, qo)


@pytest.mark.parametrize("dtype", [np.float32, np.float16])
@pytest.mark.parametrize("K,N", SHAPES)
def test_quantize_bit_exact(K, N, dtype):
    W = synthetic.weights(K, N, SEED, 1000 + K + N, outlier_frac=0.001).astype(dtype)
    _check(W)


def test_quantize_edge_columns():
    K, N = 300, 64
    W = synthetic.weights(K, N, SEED, 1100)
    W[:, 0] = 0.0                                           # all-zero column
    W[:, 1] = -0.0
    W[:, 2] = np.float32(2.0 ** -24) * np.arange(K) / K     # subnormal fp16 scale
    W[:5, 3] = np.float32(127 * 1.4 * 2.0 ** -24)           # clip engages
    W[5:, 3] = 0.0
    s0 = float(np.float16(0.0123))
    j = (np.arange(K) % 255) - 127
    W[:, 4] = (j * s0).astype(np.float32)                   # exact multiples
    W[:, 5] = np.concatenate([[127 * s0], (np.arange(K - 1) % 200 - 100 + 0.5) * s0])  # ties
    W[:, 6] = 1e-30                                         # fp32 subnormal -> zero scale
    W[7, 7] = 3.0e4                                         # one large outlier
    _check(W)


def test_quantize_16_column_strip_path():
    # K = 13696 (the ChatGLM2 4h-to-h input width) in fp32 uses 16-column strips
    W = synthetic.weights(13696, 256, SEED, 1200, outlier_frac=0.001)
    _check(W)


def test_quantize_streaming_path():
    # a strip too tall to stay in cluster shared memory is read twice
    W = synthetic.weights(30000, 72, SEED, 1300, outlier_frac=0.001)
    _check(W)


def test_quantize_repeatable():
    W = synthetic.weights(512, 264, SEED, 1400)
    a = _gpu_quant(W)
    b = _gpu_quant(W)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_quantize_chatglm2_h_to_4h_full_size():
    # 4096 x 27392 with 0.1 % outliers: every column bit-exact against the
    # oracle, plus the invariants of the pages (levels +-127, max -> 127)
    K, N = 4096, 27392
    W = synthetic.weights(K, N, SEED, synthetic.tensor_id(2, 0, 0, 0), outlier_frac=0.001)
    qg, sg = _gpu_quant(W)
    qo, so = par_quantize(W)
    assert np.array_equal(sg.view(np.uint16), so.view(np.uint16))
    assert np.array_equal(qg, qo)
    assert qg.min() >= -127 and qg.max() <= 127
    arg = np.argmax(np.abs(W), axis=0)
    assert np.all(np.abs(qg[arg, np.arange(N)]) == 127)


def test_quantize_bert_base_all_weights():
    for i, (K, N) in enumerate(synthetic.WORKLOADS["bert_base_4096_tokens"]["matrices"]):
        W = synthetic.weights(K, N, SEED, synthetic.tensor_id(5, 0, i, 0))
        _check(W)


def test_quantize_near_rounding_boundaries():
    # Each column's scale is an exact fp16 value s0 (its max is 127 * s0).
    # The other weights sit at (k + 1/2 + d) * s0 for offsets d just inside
    # and outside the band where a reciprocal-multiply and the correctly
    # rounded quotient can disagree, and at exact ties; the codes must
    # still equal those of the exact definition.
    rng = np.random.default_rng(17)
    N = 64
    offs = np.array([0.0, 2.0 ** -20, -2.0 ** -20, 2.0 ** -15, -2.0 ** -15, 2.0 ** -14, -2.0 ** -14,
                     2.0 ** -13, -2.0 ** -13, 1.5 * 2.0 ** -13, -1.5 * 2.0 ** -13, 2.0 ** -12, -2.0 ** -12,
                     1e-6, -1e-6, 3e-5, -3e-5])
    ks = np.arange(-127, 127)
    vals = (ks[:, None] + 0.5 + offs[None, :]).ravel()
    K = vals.size + 1
    W = np.empty((K, N), dtype=np.float32)
    s0 = np.float16(rng.uniform(1e-3, 8e-3, N)).astype(np.float32)
    for n in range(N):
        col = (rng.permutation(vals) * np.float64(s0[n])).astype(np.float32)
        W[0, n] = np.float32(127.0) * s0[n]
        W[1:, n] = np.clip(col, -W[0, n], W[0, n])
    _check(W)
    _check(W.astype(np.float16))
