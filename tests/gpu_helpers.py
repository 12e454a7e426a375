"""Shared helpers for the -m gpu parity tests.  Inputs come from `synthetic`
(host, seeded); the oracle only ever sees host inputs and its own outputs."""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

import oracle
import synthetic

SEED = synthetic.SEED


def torch_mod():
    import torch
    return torch


def dev():
    return torch_mod().device("cuda:0")


def to_gpu(a):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev())


def to_np(t):
    torch = torch_mod()
    torch.cuda.synchronize()
    return t.cpu().numpy()


def w8():
    import int8_weight_only_b200 as mod
    from int8_weight_only_b200 import build
    build.build()
    mod.load_library()
    return mod


def gpu_pipeline(W, X, bias=None):
    """Product path on the GPU: quantize -> prepack -> linear.
    Returns (q, scales, Y) as numpy."""
    m = w8()
    Wg = to_gpu(W)
    q, s = m.quantize(Wg)
    packed = m.prepack(q)
    Y = m.linear(to_gpu(X), packed, s, None if bias is None else to_gpu(bias))
    return to_np(q), to_np(s), to_np(Y)


def assert_close(y_gpu, y_ref, what=""):
    ok, worst = oracle.tolerance_ok(np.asarray(y_gpu, dtype=np.float64), y_ref)
    assert ok, f"{what}: worst err/bound = {worst:.3f}"
    return worst


# ---------------------------------------------------------------- the oracle on column slabs
# Every output channel is computed on its own by the oracle (quantization is
# per column, and Y[:, n] depends only on column n of q), so running the
# unchanged oracle on column slabs, concurrently, gives exactly the result it
# gives on the whole matrix, only sooner.  ctypes releases the GIL for the
# duration of each C call.
def _workers() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _slabs(N: int, width: int):
    return [(a, min(N, a + width)) for a in range(0, N, width)]


def par_quantize(W, fn=None, width: int = 1024):
    """fn(W) for one of the oracle's quantizers, on column slabs.  The first
    output (the codes, [K, N]) is joined along columns, every other output
    (per-channel vectors and [N, cap] side lists) along its first axis."""
    fn = fn or oracle.quantize
    N = W.shape[1]
    with ThreadPoolExecutor(max_workers=_workers()) as ex:
        parts = list(ex.map(lambda ab: fn(np.ascontiguousarray(W[:, ab[0]:ab[1]])), _slabs(N, width)))
    return tuple(np.concatenate([p[i] for p in parts], axis=1 if i == 0 else 0) for i in range(len(parts[0])))


def par_linear(X, q, *chan, fn=None, bias=None):
    """fn(X, q, *chan, bias) for one of the oracle's linears, on column
    slabs: q is sliced by column, every per-channel operand (scales, zero
    points, side lists, bias) by its first axis; Y is joined by column."""
    fn = fn or oracle.linear
    K, N = q.shape
    width = max(64, ((1 << 20) // max(K, 1)) // 64 * 64)

    def one(ab):
        a, b = ab
        args = [np.ascontiguousarray(c[a:b]) for c in chan]
        return fn(X, np.ascontiguousarray(q[:, a:b]), *args,
                  None if bias is None else np.ascontiguousarray(bias[a:b]))

    with ThreadPoolExecutor(max_workers=_workers()) as ex:
        parts = list(ex.map(one, _slabs(N, width)))
    return np.concatenate(parts, axis=1) if parts else np.empty((X.shape[0], 0))
