"""GPU batched quantization: one launch over many weights gives, weight by
weight, the oracle's codes and scales bit for bit (and the single-weight
entry point's)."""
import numpy as np
import pytest

import oracle
import synthetic
from tests.gpu_helpers import SEED, to_gpu, to_np, w8

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [np.float32, np.float16])
def test_batched_mixed_shapes_bit_exact(dtype):
    m = w8()
    shapes = [(768, 3072), (3072, 768), (768, 2304), (768, 768), (64, 8), (1000, 264), (13696, 136), (257, 520)]
    Ws = [synthetic.weights(K, N, SEED, 8000 + i, outlier_frac=0.001).astype(dtype) for i, (K, N) in enumerate(shapes)]
    qs, ss = m.quantize_batched([to_gpu(W) for W in Ws])
    for W, q, s in zip(Ws, qs, ss):
        qo, so = oracle.quantize(W)
        assert np.array_equal(to_np(q), qo)
        assert np.array_equal(to_np(s).view(np.uint16), so.view(np.uint16))


def test_batched_more_than_one_launch_and_equal_to_single_calls():
    # 70 weights: two launches of up to 64; every result equals the single call
    m = w8()
    rng = np.random.default_rng(9)
    shapes = [(int(rng.integers(1, 40)) * 32, int(rng.integers(1, 20)) * 8) for _ in range(70)]
    Ws = [to_gpu(synthetic.weights(K, N, SEED, 8100 + i, outlier_frac=0.01)) for i, (K, N) in enumerate(shapes)]
    qs, ss = m.quantize_batched(Ws)
    for W, q, s in zip(Ws, qs, ss):
        q1, s1 = m.quantize(W)
        assert np.array_equal(to_np(q), to_np(q1)) and np.array_equal(to_np(s), to_np(s1))


def test_batched_bert_layer_set_bit_exact():
    # the 12-layer BERT-base weight set (48 weights), checked on a sample
    m = w8()
    spec = synthetic.WORKLOADS["bert_base_4096_tokens"]
    Ws = []
    for layer in range(spec["layers"]):
        for i, (K, N) in enumerate(spec["matrices"]):
            Ws.append(synthetic.weights(K, N, SEED, synthetic.tensor_id(5, layer, i, 0)))
    qs, ss = m.quantize_batched([to_gpu(W) for W in Ws])
    for idx in (0, 5, 22, 47):
        qo, so = oracle.quantize(Ws[idx])
        assert np.array_equal(to_np(qs[idx]), qo)
        assert np.array_equal(to_np(ss[idx]).view(np.uint16), so.view(np.uint16))


def test_batched_empty_and_zero_width():
    torch = pytest.importorskip("torch")
    m = w8()
    assert m.quantize_batched([]) == ([], [])
    W = to_gpu(synthetic.weights(128, 64, SEED, 8200))
    Z = torch.zeros((16, 0), dtype=torch.float32, device="cuda")
    qs, ss = m.quantize_batched([W, Z])
    qo, so = oracle.quantize(to_np(W))
    assert np.array_equal(to_np(qs[0]), qo) and qs[1].numel() == 0
