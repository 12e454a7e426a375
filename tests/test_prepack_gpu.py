"""The packed weight layout: GPU prepack equals the layout written out in
include/w8a16.h (restated here in numpy), and unpack inverts it."""
import numpy as np
import pytest

from tests.gpu_helpers import to_gpu, to_np, w8

pytestmark = pytest.mark.gpu

SHAPES = [(64, 128), (1, 8), (65, 136), (200, 264), (4096, 4608), (13696, 264)]


def layout_reference(q):
    """Tile (b, kb) at (b*KB + kb)*8192; row r of the tile at 64r; chunk c at
    slot c ^ ((r >> 1) & 3); bytes hold q ^ 0x80; padding holds 0x80."""
    K, N = q.shape
    KB, NB = -(-K // 64), -(-N // 128)
    full = np.zeros((KB * 64, NB * 128), dtype=np.int8)
    full[:K, :N] = q
    u = (full.view(np.uint8) ^ 0x80).reshape(KB, 64, NB, 128)     # [kb, k, b, n]
    t = u.transpose(2, 0, 3, 1)                                    # [b, kb, n(r), k]
    t = t.reshape(NB, KB, 128, 4, 16)                              # chunks of 16 k
    r = np.arange(128)
    out = np.empty_like(t)
    for c in range(4):
        slot = c ^ ((r >> 1) & 3)
        out[:, :, r, slot, :] = t[:, :, r, c, :]
    return out.reshape(-1)


@pytest.mark.parametrize("K,N", SHAPES)
def test_prepack_matches_documented_layout(K, N):
    rng = np.random.default_rng(K * 7 + N)
    q = rng.integers(-127, 128, size=(K, N)).astype(np.int8)
    m = w8()
    packed = to_np(m.prepack(to_gpu(q)))
    assert packed.size == m.prepacked_bytes(K, N)
    assert np.array_equal(packed, layout_reference(q))


@pytest.mark.parametrize("K,N", SHAPES)
def test_unpack_inverts_prepack(K, N):
    rng = np.random.default_rng(K + N)
    q = rng.integers(-127, 128, size=(K, N)).astype(np.int8)
    m = w8()
    back = to_np(m.unpack(m.prepack(to_gpu(q)), K, N))
    assert np.array_equal(back, q)
