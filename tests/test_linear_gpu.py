"""GPU W8A16 linear against the oracle.

Every case runs the product pipeline on the GPU (quantize -> prepack ->
linear) and the oracle on the same host inputs (its own quantize -> fp64
linear).  Y must satisfy |Y - Y_ref| <= 2^-9 |Y_ref| + 1e-3 rms(Y_ref)
element-wise; where the arithmetic is exact, bit equality is required.
"""
import numpy as np
import pytest

import oracle
import synthetic
from tests.gpu_helpers import SEED, assert_close, gpu_pipeline, par_linear, par_quantize, to_gpu, to_np, w8

pytestmark = pytest.mark.gpu


def _case(M, K, N, tid, bias=True, outliers=0.001):
    W = synthetic.weights(K, N, SEED, tid, outlier_frac=outliers)
    X = synthetic.activations(M, K, SEED, tid + 1)
    b = synthetic.bias(N, SEED, tid + 2) if bias else None
    return W, X, b


def _check_full(M, K, N, tid, bias=True):
    W, X, b = _case(M, K, N, tid, bias)
    qg, sg, Yg = gpu_pipeline(W, X, b)
    qo, so = oracle.quantize(W)
    assert np.array_equal(qg, qo) and np.array_equal(sg.view(np.uint16), so.view(np.uint16))
    Yref = oracle.linear(X, qo, so, b)
    return assert_close(Yg, Yref, f"M={M} K={K} N={N}")


# ---------------------------------------------------------------- weight streaming (M <= 64)
DECODE_SHAPES = [(256, 512), (64, 8), (200, 136), (1024, 1032), (4096, 4608), (13696, 264)]


@pytest.mark.parametrize("M", [1, 2, 3, 8, 9, 16, 17, 31, 32, 33, 48, 64])
@pytest.mark.parametrize("K,N", DECODE_SHAPES)
def test_decode_matches_oracle(M, K, N):
    _check_full(M, K, N, 2000 + K + N + M, bias=(M % 2 == 1))


# ---------------------------------------------------------------- tensor cores (M > 64)
PREFILL_SHAPES = [(256, 512), (64, 136), (520, 264), (4096, 384)]


@pytest.mark.parametrize("M", [65, 128, 129, 256, 257, 300])
@pytest.mark.parametrize("K,N", PREFILL_SHAPES)
def test_prefill_matches_oracle(M, K, N):
    _check_full(M, K, N, 3000 + K + N + M, bias=(M % 2 == 0))


def _full(M, K, N, tid, bias=True):
    """GPU pipeline on the whole problem, every code and output checked
    against the oracle (run on column slabs in parallel)."""
    W, X, b = _case(M, K, N, tid, bias)
    qg, sg, Yg = gpu_pipeline(W, X, b)
    qo, so = par_quantize(W)
    assert np.array_equal(qg, qo) and np.array_equal(sg.view(np.uint16), so.view(np.uint16))
    assert_close(Yg, par_linear(X, qo, so, bias=b), f"M={M} K={K} N={N}")
    return Yg


def test_prefill_k_split_one_step_shares():
    # 2 pair tiles of 32 K steps: the K steps are split over 64 pairs, one
    # step each, and every tile is summed from 32 partial sums; full check
    _check_full(129, 8192, 512, 3900, bias=True)


def test_prefill_k_split_shares_cross_tiles():
    # 16 pair tiles of 32 K steps over 74 pairs: shares of 6 or 7 steps start
    # and end inside tiles (both partial-sum slots in use)
    _full(300, 8192, 2048, 3910)


def test_prefill_whole_wave_then_k_split():
    # 150 pair tiles of 32 K steps: one wave of whole tiles, then the K steps
    # of the last 76 tiles split over all pairs
    _full(3800, 8192, 2560, 3920)


def test_prefill_k_split_deterministic():
    # the split tiles' partial sums are added in K order whatever the order
    # in which the pairs finish: repeated calls agree bit for bit
    torch = pytest.importorskip("torch")
    m = w8()
    W, X, b = _case(300, 8192, 2048, 3930)
    q, s = m.quantize(to_gpu(W))
    packed = m.prepack(q)
    Xg, bg = to_gpu(X), to_gpu(b)
    Y1 = to_np(m.linear(Xg, packed, s, bg))
    for _ in range(3):
        Y2 = to_np(m.linear(Xg, packed, s, bg))
        assert np.array_equal(Y1.view(np.uint16), Y2.view(np.uint16))


def test_prefill_whole_waves_ragged_tail():
    # 190 pair tiles of 2 K steps: three waves of whole tiles, the last one
    # partly filled
    _full(1280, 512, 9728, 3950)


def test_tiny_workload_both_paths():
    # 4 x 256 activations, 256 x 512 weight (the smallest workload), then the
    # same weight through the tensor-core path with 4 copies of X stacked
    _check_full(4, 256, 512, synthetic.tensor_id(1, 0, 0, 0), bias=False)
    W, X, _ = _case(4, 256, 512, synthetic.tensor_id(1, 0, 0, 0), bias=False)
    X32 = np.concatenate([X] * 8, axis=0)
    qg, sg, Yg = gpu_pipeline(W, X32)
    qo, so = oracle.quantize(W)
    assert_close(Yg, oracle.linear(X32, qo, so), "stacked")


# ---------------------------------------------------------------- exact cases
@pytest.mark.parametrize("M", [1, 5, 16, 40, 200])
def test_exact_integer_inputs_bit_exact(M):
    # integer X and power-of-two-multiple weights: every product and partial
    # sum is exact in fp32, so Y must equal the exact value rounded to fp16
    rng = np.random.default_rng(M)
    K, N = 512, 264
    X = rng.integers(-8, 9, size=(M, K)).astype(np.float16)
    s0 = 2.0 ** rng.integers(-10, -4, size=N)
    j = rng.integers(-127, 128, size=(K, N))
    j[0] = 127
    W = (j * s0).astype(np.float32)
    b = (rng.integers(-64, 64, size=N) / 16.0).astype(np.float16)
    qg, sg, Yg = gpu_pipeline(W, X, b)
    qo, so = oracle.quantize(W)
    Yref = oracle.linear(X, qo, so, b)
    assert np.array_equal(Yg.view(np.uint16), Yref.astype(np.float16).view(np.uint16))


def test_unit_rows_select_weight_rows():
    K, N = 320, 136
    W, _, _ = _case(1, K, N, 3500, bias=False)
    ks = [0, 63, 64, 319]
    for M in (len(ks), 32):
        X = np.zeros((M, K), dtype=np.float16)
        for m in range(M):
            X[m, ks[m % len(ks)]] = 1.0
        qg, sg, Yg = gpu_pipeline(W, X)
        qo, so = oracle.quantize(W)
        Yref = oracle.linear(X, qo, so)
        assert np.array_equal(Yg.view(np.uint16), Yref.astype(np.float16).view(np.uint16))


def test_deterministic_across_calls():
    m = w8()
    for M in (1, 16, 100):
        W, X, b = _case(M, 2048, 1024, 3600 + M)
        q, s = m.quantize(to_gpu(W))
        packed = m.prepack(q)
        Xg, bg = to_gpu(X), to_gpu(b)
        Y1 = to_np(m.linear(Xg, packed, s, bg))
        Y2 = to_np(m.linear(Xg, packed, s, bg))
        assert np.array_equal(Y1.view(np.uint16), Y2.view(np.uint16))


def test_workspace_reused_across_shapes():
    # the split-K counters are reset by each call, so one workspace serves
    # calls of different shapes and token counts back to back, weight
    # streaming and tensor-core paths alike
    for (M, K, N) in [(1, 4096, 512), (3, 64, 8), (16, 1000, 1032), (64, 2048, 4104), (1, 4096, 512),
                      (300, 8192, 2048), (40, 4096, 27392), (129, 8192, 512), (9, 13696, 264),
                      (129, 8192, 512)]:
        _check_full(M, K, N, 3700 + K + N)


def test_workspace_too_small_is_rejected():
    torch = pytest.importorskip("torch")
    m = w8()
    W, X, _ = _case(1, 256, 512, 3800)
    q, s = m.quantize(to_gpu(W))
    packed = m.prepack(q)
    need = m.workspace_bytes(1, 256, 512)
    assert need > 0
    ws = torch.zeros(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(m.W8Error) as e:
        m.linear(to_gpu(X), packed, s, workspace=ws)
    assert e.value.status == -5
    # one layout for every token count: the K-split partial sums of both kernels
    assert m.workspace_bytes(65, 256, 512) == m.workspace_bytes(64, 256, 512) > 0
    assert m.workspace_bytes(0, 256, 512) == 0


def test_empty_batch():
    torch = pytest.importorskip("torch")
    m = w8()
    W, _, _ = _case(1, 64, 128, 3900)
    q, s = m.quantize(to_gpu(W))
    packed = m.prepack(q)
    Y = m.linear(torch.zeros((0, 64), dtype=torch.float16, device="cuda"), packed, s)
    assert tuple(Y.shape) == (0, 128)

# The full-size workloads (every output of every config) are checked in
# test_full_size_gpu.py.


def test_default_workspace_per_stream():
    # calls without workspace= on two streams may overlap on the GPU, so
    # each stream gets its own default split-K scratch; results on both
    # streams, launched interleaved, must match the oracle
    torch = pytest.importorskip("torch")
    m = w8()
    shapes = [(1, 4096, 4608), (16, 13696, 4096)]
    cases = []
    for i, (M, K, N) in enumerate(shapes):
        W, X, b = _case(M, K, N, 4100 + i)
        q, s = m.quantize(to_gpu(W))
        cases.append((W, X, b, m.prepack(q), s, to_gpu(X), to_gpu(b)))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [[], []]
    for rep in range(8):
        for j, st in enumerate(streams):
            W, X, b, packed, s, Xg, bg = cases[j]
            with torch.cuda.stream(st):
                outs[j].append(m.linear(Xg, packed, s, bg))
    torch.cuda.synchronize()
    keys = {k for k in m._ws_cache if k[1] in (streams[0].cuda_stream, streams[1].cuda_stream)}
    assert len(keys) == 2
    for j in range(2):
        W, X, b = cases[j][:3]
        qo, so = oracle.quantize(W)
        Yref = oracle.linear(X, qo, so, b)
        for Y in outs[j]:
            assert_close(to_np(Y), Yref, f"stream {j}")
