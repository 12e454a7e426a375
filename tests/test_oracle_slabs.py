"""The parity tests run the oracle on column slabs in parallel.  Each output
channel is independent, so this must reproduce the oracle's whole-matrix
result exactly; checked here for every quantizer and linear, with a slab
width that leaves a ragged last slab."""
import numpy as np

import oracle
import synthetic
from tests.gpu_helpers import par_linear, par_quantize

SEED = synthetic.SEED


def _inputs(K=200, N=1000, M=5):
    W = synthetic.weights(K, N, SEED, 8800, outlier_frac=0.01)
    X = synthetic.activations(M, K, SEED, 8801)
    b = synthetic.bias(N, SEED, 8802)
    return W, X, b


def _same(a, b):
    assert len(a) == len(b)
    for x, y in zip(a, b):
        assert x.dtype == y.dtype and np.array_equal(x.view(np.uint8), y.view(np.uint8))


def test_slabbed_symmetric():
    W, X, b = _inputs()
    whole = oracle.quantize(W)
    _same(par_quantize(W, width=96), whole)
    q, s = whole
    Y = par_linear(X, q, s, bias=b)
    assert np.array_equal(Y, oracle.linear(X, q, s, b))


def test_slabbed_asymmetric():
    W, X, b = _inputs()
    whole = oracle.quantize_asym(W)
    _same(par_quantize(W, fn=oracle.quantize_asym, width=96), whole)
    assert np.array_equal(par_linear(X, *whole, fn=oracle.linear_asym, bias=b), oracle.linear_asym(X, *whole, b))


def test_slabbed_outliers():
    W, X, b = _inputs()
    whole = oracle.quantize_outliers(W, 0.97)
    _same(par_quantize(W, fn=lambda w: oracle.quantize_outliers(w, 0.97), width=96), whole)
    assert np.array_equal(par_linear(X, *whole, fn=oracle.linear_outliers, bias=b),
                          oracle.linear_outliers(X, *whole, bias=b))
