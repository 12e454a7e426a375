"""Full-size parity on every workload: every code, scale and output checked.

The workloads are the pages' shapes (TPU-MLIR ChatGLM2 W8A16 article,
section 3, the 4096 x 27392 weight, and section 4, figure "MatMuls in
ChatGLM2 prefill and decode phase"; the LightSeq article's BERT-base
configuration with 4096 batch tokens), filled with the seeded synthetic
values the benchmark uses.  For each distinct weight the GPU's codes and
scales must equal the oracle's bit for bit on every column, and every
element of Y must satisfy |Y - Y_ref| <= 2^-9 |Y_ref| + 1e-3 rms(Y_ref)
against the oracle's fp64 product.  The oracle runs unchanged, on column
slabs in parallel (see ``gpu_helpers.par_quantize``), which gives its
whole-matrix result.
"""
import functools

import numpy as np
import pytest

import oracle
import synthetic
from tests.gpu_helpers import SEED, assert_close, par_linear, par_quantize, to_gpu, to_np, w8

pytestmark = pytest.mark.gpu

WL = synthetic.WORKLOADS

# (name, K, N, weight tensor id, outlier fraction): every distinct weight of
# the five workloads
WEIGHTS = (
    [("tiny", 256, 512, synthetic.tensor_id(1, 0, 0, 0), 0.0),
     ("h_to_4h_decode", 4096, 27392, synthetic.tensor_id(2, 0, 0, 0), 0.001)]
    + [(f"decode_set_{i}", K, N, synthetic.tensor_id(3, 0, i, 0), WL["chatglm2_decode_set"]["outlier_frac"])
       for i, (K, N) in enumerate(WL["chatglm2_decode_set"]["matrices"])]
    + [(f"prefill_{i}", K, N, synthetic.tensor_id(4, 0, i, 0), WL["chatglm2_prefill"]["outlier_frac"])
       for i, (K, N) in enumerate(WL["chatglm2_prefill"]["matrices"])]
    + [(f"bert_{i}", K, N, synthetic.tensor_id(5, 0, i, 0), 0.0)
       for i, (K, N) in enumerate(WL["bert_base_4096_tokens"]["matrices"])]
)
BY_NAME = {w[0]: w for w in WEIGHTS}


@functools.lru_cache(maxsize=2)
def _weight(name):
    """(W host, oracle q, oracle scales) of one workload weight."""
    _, K, N, tid, frac = BY_NAME[name]
    W = synthetic.weights(K, N, SEED, tid, outlier_frac=frac)
    q, s = par_quantize(W)
    return W, q, s


def _gpu_weight(name):
    """GPU codes, scales and packed tiles; codes and scales checked against
    the oracle on every column."""
    m = w8()
    W, qo, so = _weight(name)
    q, s = m.quantize(to_gpu(W))
    packed = m.prepack(q)
    qg, sg = to_np(q), to_np(s)
    assert np.array_equal(sg.view(np.uint16), so.view(np.uint16)), f"{name}: scales differ"
    bad = np.argwhere(qg != qo)
    assert bad.size == 0, f"{name}: {len(bad)} codes differ, first at (k, n) = {tuple(bad[0])}"
    return packed, s


@pytest.mark.parametrize("name", [w[0] for w in WEIGHTS])
def test_quantize_every_column(name):
    _gpu_weight(name)


@pytest.mark.parametrize("dtype", [np.float32, np.float16])
def test_quantize_h_to_4h_fp16_and_fp32_agree(dtype):
    # the page's R is f16; widening it is exact, so fp16 storage of the same
    # values gives the same codes as the fp32 path and as the oracle
    m = w8()
    W, _, _ = _weight("h_to_4h_decode")
    W16 = W.astype(np.float16)
    Wd = W16 if dtype == np.float16 else W16.astype(np.float32)
    q, s = m.quantize(to_gpu(Wd))
    qo, so = par_quantize(W16)
    assert np.array_equal(to_np(s).view(np.uint16), so.view(np.uint16))
    assert np.array_equal(to_np(q), qo)


def test_h_to_4h_decode_every_output():
    # the headline call: M = 1, 4096 x 27392, 0.1 % outliers
    m = w8()
    packed, s = _gpu_weight("h_to_4h_decode")
    _, qo, so = _weight("h_to_4h_decode")
    tid = synthetic.tensor_id(2, 0, 0, 0)
    X = synthetic.activations(1, 4096, SEED, tid + 1)
    Y = to_np(m.linear(to_gpu(X), packed, s))
    assert_close(Y, par_linear(X, qo, so), "h-to-4h decode M=1")


@pytest.mark.parametrize("i", range(len(WL["chatglm2_decode_set"]["matrices"])))
def test_decode_set_every_output(i):
    # every token count of the decode set (and the decode kernel's upper
    # range, 32 and 64 tokens) on each of the four ChatGLM2 layer weights
    m = w8()
    name = f"decode_set_{i}"
    packed, s = _gpu_weight(name)
    _, qo, so = _weight(name)
    K, N = BY_NAME[name][1], BY_NAME[name][2]
    for M in (1, 2, 4, 8, 16, 32, 64):
        X = synthetic.activations(M, K, SEED, synthetic.tensor_id(3, M, i, 1))
        b = synthetic.bias(N, SEED, synthetic.tensor_id(3, M, i, 2)) if M % 4 == 2 else None
        Y = to_np(m.linear(to_gpu(X), packed, s, None if b is None else to_gpu(b)))
        assert_close(Y, par_linear(X, qo, so, bias=b), f"{name} M={M}")


@pytest.mark.parametrize("M", WL["chatglm2_prefill"]["M"])
@pytest.mark.parametrize("i", range(len(WL["chatglm2_prefill"]["matrices"])))
def test_prefill_every_output(i, M):
    m = w8()
    name = f"prefill_{i}"
    packed, s = _gpu_weight(name)
    _, qo, so = _weight(name)
    K = BY_NAME[name][1]
    X = synthetic.activations(M, K, SEED, synthetic.tensor_id(4, M, i, 1))
    Y = to_np(m.linear(to_gpu(X), packed, s))
    assert_close(Y, par_linear(X, qo, so), f"{name} M={M}")


@pytest.mark.parametrize("i", range(len(WL["bert_base_4096_tokens"]["matrices"])))
def test_bert_base_4096_tokens_every_output(i):
    m = w8()
    name = f"bert_{i}"
    packed, s = _gpu_weight(name)
    _, qo, so = _weight(name)
    K, N, tid = BY_NAME[name][1], BY_NAME[name][2], BY_NAME[name][3]
    X = synthetic.activations(4096, K, SEED, tid + 1)
    b = synthetic.bias(N, SEED, tid + 2)
    Y = to_np(m.linear(to_gpu(X), packed, s, to_gpu(b)))
    assert_close(Y, par_linear(X, qo, so, bias=b), f"{name} M=4096")


def test_bert_base_batched_quantize_every_column():
    # all four BERT-base weight shapes in one launch, against the oracle
    m = w8()
    Ws = [_weight_direct(f"bert_{i}") for i in range(4)]
    qs, ss = m.quantize_batched([to_gpu(W) for W in Ws])
    for W, q, s in zip(Ws, qs, ss):
        qo, so = oracle.quantize(W)
        assert np.array_equal(to_np(s).view(np.uint16), so.view(np.uint16))
        assert np.array_equal(to_np(q), qo)


def _weight_direct(name):
    _, K, N, tid, frac = BY_NAME[name]
    return synthetic.weights(K, N, SEED, tid, outlier_frac=frac)
