"""Seeded synthetic inputs for the W8A16 linear layer.

This module is shared by the CPU oracle's tests, the GPU parity tests and
the benchmark.  It holds no quantization or GEMM arithmetic: it only turns
(seed, tensor id, element index) into numbers, so both sides of every parity
check start from identical bytes.

Generator (counter based, so any element can be drawn on its own):

* ``splitmix64`` finaliser ``mix(z)`` (Steele, Lea and Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014).
* Stream key ``key = mix(seed + G*(tensor_id + 1))`` with
  ``G = 0x9E3779B97F4A7C15`` (all arithmetic modulo 2**64).
* Element ``i`` draws two 64-bit words ``a = mix(key + G*(2i+1))`` and
  ``b = mix(key + G*(2i+2))``, maps them to ``u1 = ((a>>11)+1)*2**-53`` in
  (0, 1] and ``u2 = (b>>11)*2**-53`` in [0, 1), and applies the Box-Muller
  transform ``z = sqrt(-2 ln u1) * cos(2 pi u2)`` (Box and Muller, 1958).
* Outliers use an independent stream ``key2 = mix(key ^ 0xD1B54A32D192ED03)``;
  element ``i`` is an outlier when ``mix(key2 + G*(i+1)) < frac * 2**64``.

Value statistics follow the pages' workloads: weights are Gaussian with
sigma 0.02 and, where a workload asks for it, 0.1 % of entries replaced by
outliers drawn with a 10x larger sigma (GOBO review, "proposed method":
99.9 % of a layer's weights are Gaussian, 0.1 % are outliers); activations
are N(0, 1) rounded to fp16.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

__all__ = [
    "GOLDEN",
    "mix64",
    "stream_key",
    "normal",
    "outlier_mask",
    "weights",
    "activations",
    "bias",
    "tensor_id",
    "WORKLOADS",
]

GOLDEN = 0x9E3779B97F4A7C15
_M64 = (1 << 64) - 1
_OUTLIER_SALT = 0xD1B54A32D192ED03
_CHUNK = 1 << 21


def _mix_scalar(z: int) -> int:
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def mix64(z: np.ndarray) -> np.ndarray:
    """splitmix64 finaliser on a uint64 array (wrapping arithmetic)."""
    z = z ^ (z >> np.uint64(30))
    z = z * np.uint64(0xBF58476D1CE4E5B9)
    z = z ^ (z >> np.uint64(27))
    z = z * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tid: int) -> int:
    return _mix_scalar((seed + GOLDEN * (tid + 1)) & _M64)


def _normal_chunk(key: int, start: int, count: int) -> np.ndarray:
    i = np.arange(start, start + count, dtype=np.uint64)
    base = np.uint64(key)
    g = np.uint64(GOLDEN)
    two_i = i * np.uint64(2)
    a = mix64(base + g * (two_i + np.uint64(1)))
    b = mix64(base + g * (two_i + np.uint64(2)))
    u1 = ((a >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * 2.0 ** -53
    u2 = (b >> np.uint64(11)).astype(np.float64) * 2.0 ** -53
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def _outlier_chunk(key: int, start: int, count: int, thresh: int) -> np.ndarray:
    key2 = _mix_scalar(key ^ _OUTLIER_SALT)
    i = np.arange(start, start + count, dtype=np.uint64)
    h = mix64(np.uint64(key2) + np.uint64(GOLDEN) * (i + np.uint64(1)))
    return h < np.uint64(thresh)


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _parallel_fill(out_flat: np.ndarray, fn) -> None:
    n = out_flat.size
    starts = list(range(0, n, _CHUNK))

    def work(s):
        c = min(_CHUNK, n - s)
        out_flat[s:s + c] = fn(s, c)

    if len(starts) <= 1:
        for s in starts:
            work(s)
        return
    with ThreadPoolExecutor(max_workers=_threads()) as ex:
        list(ex.map(work, starts))


def normal(seed: int, tid: int, n: int) -> np.ndarray:
    """n standard-normal float64 draws of stream (seed, tid), elements 0..n-1."""
    key = stream_key(seed, tid)
    out = np.empty(n, dtype=np.float64)
    _parallel_fill(out, lambda s, c: _normal_chunk(key, s, c))
    return out


def outlier_mask(seed: int, tid: int, n: int, frac: float) -> np.ndarray:
    key = stream_key(seed, tid)
    thresh = int(frac * 2.0 ** 64)
    out = np.empty(n, dtype=np.bool_)
    _parallel_fill(out, lambda s, c: _outlier_chunk(key, s, c, thresh))
    return out


def weights(K: int, N: int, seed: int, tid: int, sigma: float = 0.02,
            outlier_frac: float = 0.0, outlier_sigma: float = 0.2,
            dtype=np.float32) -> np.ndarray:
    """Weight matrix W[K, N] (row-major, N contiguous).

    Gaussian N(0, sigma^2); with ``outlier_frac > 0`` that fraction of
    entries (chosen by the independent outlier stream) is drawn from
    N(0, outlier_sigma^2) instead, reusing the element's own normal draw.
    """
    n = K * N
    key = stream_key(seed, tid)
    thresh = int(outlier_frac * 2.0 ** 64)
    out = np.empty(n, dtype=dtype)

    def fn(s, c):
        z = _normal_chunk(key, s, c)
        if outlier_frac > 0.0:
            m = _outlier_chunk(key, s, c, thresh)
            return np.where(m, z * outlier_sigma, z * sigma).astype(dtype)
        return (z * sigma).astype(dtype)

    _parallel_fill(out, fn)
    return out.reshape(K, N)


def activations(M: int, K: int, seed: int, tid: int, sigma: float = 1.0) -> np.ndarray:
    """Activations X[M, K] fp16: N(0, sigma^2) rounded to nearest fp16."""
    z = normal(seed, tid, M * K) * sigma
    return z.astype(np.float16).reshape(M, K)


def bias(N: int, seed: int, tid: int, sigma: float = 0.1) -> np.ndarray:
    """Optional per-channel bias b[N] fp16."""
    return (normal(seed, tid, N) * sigma).astype(np.float16)


def tensor_id(workload: int, layer: int, matrix: int, role: int) -> int:
    """Distinct stream id per (workload, layer, matrix, role).

    role: 0 = weight, 1 = activation, 2 = bias.
    """
    return ((workload * 1000 + layer) * 100 + matrix) * 10 + role


# Shapes of the pages' workloads (TPU-MLIR W8A16 article: the ChatGLM2-6B
# GLMBlock linears, "TPU-MLIR implementation" and "backend performance"
# sections; LightSeq article: BERT-base configuration with 4096 batch tokens).
# Each entry: (K, N) per matrix, the token counts M, and value statistics.
WORKLOADS = {
    "tiny": {
        "matrices": [(256, 512)],
        "M": [4],
        "outlier_frac": 0.0,
        "layers": 1,
    },
    "chatglm2_h_to_4h_decode": {
        "matrices": [(4096, 27392)],
        "M": [1],
        "outlier_frac": 0.001,
        "layers": 1,
    },
    "chatglm2_decode_set": {
        "matrices": [(4096, 4608), (4096, 4096), (4096, 27392), (13696, 4096)],
        "M": [1, 2, 4, 8, 16],
        "outlier_frac": 0.001,
        "layers": 28,
    },
    "chatglm2_prefill": {
        "matrices": [(4096, 27392), (13696, 4096)],
        "M": [512, 1024, 2048],
        "outlier_frac": 0.001,
        "layers": 1,
    },
    "bert_base_4096_tokens": {
        "matrices": [(768, 3072), (3072, 768), (768, 2304), (768, 768)],
        "M": [4096],
        "outlier_frac": 0.0,
        "layers": 12,
    },
}

SEED = 20231002
