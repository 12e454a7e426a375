"""Decode split-K bookkeeping: the paths that timing rarely takes give the
same bits as the usual ones.

A channel block whose K range is split between CTAs is finished by one of
them from fp32 partial sums added in CTA order.  Normally the CTA that
streams the block's first K blocks last picks up the next CTA's part
during its stream (or the last of several contributors adds all parts).
The test hook delays each CTA's count of the part it publishes for its
first block, so the next-CTA look fails, the previous CTA takes the
general path without being last, and the delayed CTA finishes its first
block after its own stream.  The parts are added in the same order on
every path, so Y must be bit-identical, and the workspace counters must
be left at zero (the next undelayed call is identical too)."""
import numpy as np
import pytest

import synthetic
from tests.gpu_helpers import assert_close, par_linear, par_quantize, to_gpu, to_np, torch_mod, w8

pytestmark = pytest.mark.gpu

# (M, K, N): two-way splits (the ChatGLM2 h-to-4h shape), splits over many
# CTAs (long K, few channel blocks), ragged K and N, up to 64 tokens.  Up to
# 16 tokens on few channel blocks the kernel's cluster form runs instead (no
# shared counters: test_decode_cluster_gpu.py), so those shapes are taken
# with more tokens or more channel blocks here.
SHAPES = [(1, 4096, 27392), (20, 13696, 4096), (40, 4096, 4096), (64, 4096, 4608), (3, 1000, 16392),
          (1, 8192, 1024), (16, 13696, 11008)]
DELAY_NS = 200_000


def mid_stream_publishers(K, N, sms):
    """CTAs whose first channel block starts past K block 0 and that have
    more work after it (the ones the hook delays), for the kernel's split of
    the T = ceil(N/128) * ceil(K/64) tiles into G = min(SMs, T) equal
    contiguous ranges."""
    KB, NB = -(-K // 64), -(-N // 128)
    T = NB * KB
    G = min(sms, T)
    out = []
    for i in range(G):
        tb, te = i * T // G, (i + 1) * T // G
        if tb % KB != 0 and (tb // KB + 1) * KB < te:
            out.append(i)
    return out


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_delayed_count_gives_identical_bits(M, K, N):
    torch = torch_mod()
    m = w8()
    assert mid_stream_publishers(K, N, torch.cuda.get_device_properties(0).multi_processor_count)
    tid = 7000 + 10 * SHAPES.index((M, K, N))
    W = synthetic.weights(K, N, synthetic.SEED, tid, outlier_frac=0.001)
    X = synthetic.activations(M, K, synthetic.SEED, tid + 1)
    bias = synthetic.bias(N, synthetic.SEED, tid + 2)
    q, s = m.quantize(to_gpu(W))
    packed = m.prepack(q)
    Xg, bg = to_gpu(X), to_gpu(bias)
    y0 = m.linear(Xg, packed, s, bg)
    torch.cuda.synchronize()
    assert m.device_status() == 0

    m.test_set_decode_helper_delay(DELAY_NS)
    try:
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        y1 = m.linear(Xg, packed, s, bg)
        stop.record()
        torch.cuda.synchronize()
        delayed_us = start.elapsed_time(stop) * 1e3
    finally:
        m.test_set_decode_helper_delay(0)
    assert m.device_status() == 0
    # the hook took effect (some CTA waited the delay before counting)
    assert delayed_us > 0.5 * DELAY_NS / 1e3, delayed_us

    y2 = m.linear(Xg, packed, s, bg)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    assert torch.equal(y0, y1), "delayed count changed Y"
    assert torch.equal(y0, y2), "counters not left at zero"

    # and the result is right: every output against the oracle
    qo, so = par_quantize(W)
    assert np.array_equal(to_np(q), qo)
    assert_close(to_np(y0), par_linear(X, qo, so, bias=bias), f"M={M} K={K} N={N}")
