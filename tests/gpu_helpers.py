"""Shared helpers for the -m gpu parity tests.  Inputs come from `synthetic`
(host, seeded); the oracle only ever sees host inputs and its own outputs."""
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
