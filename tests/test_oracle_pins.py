"""Pins for the CPU oracle: checks against what the pages and mathematics fix,
never against a retyped copy of the oracle's own formula.

Sources: TPU-MLIR ChatGLM2 W8A16 article (sections 2-4) and LightSeq 2020
slides ("quantization: clipping + symmetric").
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synthetic
from tests import golden

SEED = synthetic.SEED


# ---------------------------------------------------------------- fp16 codec
# Pinned to numpy's IEEE binary16 conversion (a library routine).

def pin_f16_to_f32_every_pattern(orc):
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = orc.f16_bits_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def pin_f32_to_f16_round_trips_every_fp16_value(orc):
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = h.view(np.float16)
    keep = ~np.isnan(f)
    back = orc.f32_to_f16_bits(f[keep].astype(np.float32))
    assert np.array_equal(back, h[keep])


def pin_f32_to_f16_ties_go_to_even(orc):
    # midpoints between adjacent finite fp16 values (exact in fp32)
    h = np.arange(0, 0x7BFF, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)
    got = orc.f32_to_f16_bits(mid)
    assert np.all(got % 2 == 0)                     # even significand
    assert np.all((got == h) | (got == h + 1))
    assert np.array_equal(got, mid.astype(np.float16).view(np.uint16))
    got_neg = orc.f32_to_f16_bits(-mid)
    assert np.array_equal(got_neg, got | np.uint16(0x8000))


def pin_f32_to_f16_random_against_numpy(orc):
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 1 << 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    # also a dense sample around the fp16 range, including fp16 subnormals
    g = (rng.standard_normal(1_000_000) * np.exp(rng.uniform(-20, 12, 1_000_000))).astype(np.float32)
    for x in (f, g):
        got = orc.f32_to_f16_bits(x)
        ref = x.astype(np.float16).view(np.uint16)
        assert np.array_equal(got, ref)


# ------------------------------------------------------------ quantization

def _wq(K, N, tid, outliers=0.001):
    return synthetic.weights(K, N, SEED, tid, outlier_frac=outliers)


def pin_symmetric_levels_from_slides(orc):
    g = golden.load("symmetric_levels.txt")
    top = 2 ** (g["bits"] - 1) - 1
    assert top == g["top_level"] == 127
    W = _wq(300, 264, 11)
    q, s = orc.quantize(W)
    assert q.min() >= -top and q.max() <= top
    assert not np.any(q == -128)
    # the bound max|W| of every channel lands on the top level, with its sign
    arg = np.argmax(np.abs(W), axis=0)
    cols = np.arange(W.shape[1])
    assert np.all(np.abs(q[arg, cols]) == top)
    assert np.all(np.sign(q[arg, cols]) == np.sign(W[arg, cols]))


def pin_error_bound_half_a_step(orc):
    # |w - q s| <= s/2, up to the single fp32 rounding of w/s
    for tid, (K, N) in enumerate([(300, 264), (64, 8), (1, 16), (1000, 40)]):
        W = _wq(K, N, 20 + tid)
        q, s = orc.quantize(W)
        s64 = s.astype(np.float64)
        err = np.abs(W.astype(np.float64) - q.astype(np.float64) * s64)
        assert np.all(err <= s64 * (0.5 + 2.0 ** -16))


def pin_scale_is_fp16_of_fp32_amax_over_127(orc):
    # library pin: numpy fp32 division (IEEE) then numpy fp16 rounding
    W = _wq(257, 72, 30)
    _, s = orc.quantize(W)
    amax = np.max(np.abs(W), axis=0).astype(np.float32)
    ref = (amax / np.float32(127.0)).astype(np.float16)
    assert np.array_equal(s.view(np.uint16), ref.view(np.uint16))


def pin_exact_multiples_round_trip(orc):
    rng = np.random.default_rng(5)
    K, N = 200, 12
    for s0 in [2.0 ** -10, 0.0004506, 1.5e-3, 0.0078125, 3.0]:
        s0 = float(np.float16(s0))
        j = rng.integers(-127, 128, size=(K, N))
        j[rng.integers(0, K, size=N), np.arange(N)] = rng.choice([-127, 127], size=N)
        W = (j * s0).astype(np.float32)
        assert np.array_equal(W.astype(np.float64), j * s0)        # exact
        q, s = orc.quantize(W)
        assert np.all(s.astype(np.float64) == s0)
        assert np.array_equal(q.astype(np.int64), j)


def pin_ties_round_half_to_even(orc):
    js = np.arange(-126, 126)
    for s0 in [2.0 ** -8, float(np.float16(0.0123))]:
        col = np.concatenate([[127.0 * s0], (js + 0.5) * s0]).astype(np.float32)
        assert np.array_equal(col[1:].astype(np.float64), (js + 0.5) * s0)
        q, s = orc.quantize(col.reshape(-1, 1))
        assert float(s[0]) == s0
        got = q[1:, 0].astype(np.int64)
        want = np.where(js % 2 == 0, js, js + 1)         # nearest even integer
        assert np.array_equal(got, want)


def pin_subnormal_scale_clamps_to_symmetric_range(orc):
    # A channel whose scale is an fp16 subnormal is coarsely rounded: here
    # s32 = 1.4 * 2^-24 rounds to s = 2^-24, so amax/s is about 178 and the
    # clip must hold the codes at +-127 (never -128).
    amax = np.float32(127 * 1.4 * 2.0 ** -24)
    col = np.array([amax, -amax, amax / 2, np.float32(3 * 2.0 ** -24)], dtype=np.float32)
    q, s = orc.quantize(np.stack([col, -col], axis=1))
    assert np.all(s.view(np.uint16) == 1)                  # 2^-24
    assert q[0, 0] == 127 and q[1, 0] == -127 and q[0, 1] == -127 and q[1, 1] == 127
    assert q[3, 0] == 3 and q[3, 1] == -3


def pin_zero_column_has_zero_scale_and_codes(orc):
    W = _wq(64, 16, 40)
    W[:, 3] = 0.0
    W[:, 9] = -0.0
    q, s = orc.quantize(W)
    assert s.view(np.uint16)[3] == 0 and s.view(np.uint16)[9] == 0
    assert not np.any(q[:, 3]) and not np.any(q[:, 9])


def pin_divides_by_the_stored_fp16_scale(orc):
    # Reading of the pages: the weights are divided by the scale that is
    # stored (fp16), so that q*s reconstructs w within s/2 for the shipped s.
    amax = np.float32(1.0)
    s32 = amax / np.float32(127.0)
    s16 = np.float32(np.float16(s32))
    assert s16 != s32
    w = np.float32(100.502) * s16
    by16 = np.rint(w / s16)
    by32 = np.rint(w / s32)
    assert by16 != by32                         # the case distinguishes them
    q, s = orc.quantize(np.array([[amax], [w]], dtype=np.float32))
    assert np.float32(s[0]) == s16
    assert q[1, 0] == by16


def pin_per_channel_independence(orc):
    W = _wq(128, 32, 50)
    q, s = orc.quantize(W)
    W2 = W.copy()
    W2[:, 5] *= np.float32(4.0)                 # power of two: exact
    q2, s2 = orc.quantize(W2)
    assert np.array_equal(q, q2)
    assert float(s2[5]) == 4.0 * float(s[5])
    keep = np.arange(32) != 5
    assert np.array_equal(s[keep].view(np.uint16), s2[keep].view(np.uint16))


def pin_fp16_weights_match_widened_fp32(orc):
    W16 = _wq(96, 40, 60).astype(np.float16)
    qa, sa = orc.quantize(W16)
    qb, sb = orc.quantize(W16.astype(np.float32))
    assert np.array_equal(qa, qb)
    assert np.array_equal(sa.view(np.uint16), sb.view(np.uint16))


def pin_codes_are_the_nearest_level_by_brute_force(orc):
    # Independent characterisation: among all 255 levels, q is the one
    # nearest to the fp32 quotient w/s (ties to the even level).
    W = _wq(9, 6, 70)
    q, s = orc.quantize(W)
    for n in range(W.shape[1]):
        sn = np.float32(s[n])
        for k in range(W.shape[0]):
            r = Fraction(float(np.float32(W[k, n]) / sn))
            best = None
            for lv in range(-127, 128):
                d = abs(r - lv)
                if best is None or d < best[0] or (d == best[0] and lv % 2 == 0):
                    best = (d, lv)
            assert q[k, n] == best[1]


def pin_weight_bytes_halve_as_printed(orc):
    g = golden.load("chatglm2_h_to_4h_weight_bytes.txt")
    K, N = g["K"], g["N"]
    f16_bytes = K * N * np.dtype(np.float16).itemsize
    # quantized storage of a small slab scales linearly: 1 byte per weight
    q, s = orc.quantize(_wq(64, 128, 80))
    per_weight = q.nbytes / q.size
    int8_bytes = K * N * per_weight
    assert round(f16_bytes / 2 ** 20) == g["f16_mb"]
    assert round(int8_bytes / 2 ** 20) == g["int8_mb"]
    # the printed scale vector has 4096 f16 entries = 0.008 MB
    assert round(g["scale_entries_printed"] * 2 / 2 ** 20, 3) == g["scale_mb_printed"]
    # one fp16 scale per output channel (the reading used here) costs N*2
    # bytes, still well under 0.1 % of the int8 weight
    scale_bytes = N * s.itemsize
    assert scale_bytes / int8_bytes < 1e-3


# ------------------------------------------------------------------ linear

def pin_linear_exact_on_integer_inputs(orc):
    # Integer X, power-of-two scales: the exact result is an integer matmul
    # (numpy int64) times the scale, with no rounding anywhere.
    rng = np.random.default_rng(7)
    M, K, N = 5, 96, 40
    Xi = rng.integers(-8, 9, size=(M, K))
    qi = rng.integers(-127, 128, size=(K, N)).astype(np.int8)
    s = (2.0 ** rng.integers(-12, -2, size=N)).astype(np.float16)
    b = (rng.integers(-64, 64, size=N) / 16.0).astype(np.float16)
    Y = orc.linear(Xi.astype(np.float16), qi, s, b)
    exact = (Xi @ qi.astype(np.int64)) * s.astype(np.float64) + b.astype(np.float64)
    assert np.array_equal(Y, exact)
    Y0 = orc.linear(Xi.astype(np.float16), qi, s, None)
    assert np.array_equal(Y0, (Xi @ qi.astype(np.int64)) * s.astype(np.float64))


def pin_linear_unit_vectors_select_rows(orc):
    rng = np.random.default_rng(8)
    K, N = 33, 24
    q = rng.integers(-127, 128, size=(K, N)).astype(np.int8)
    s = (rng.uniform(1e-4, 1e-2, N)).astype(np.float16)
    ks = [0, 7, 32]
    X = np.zeros((len(ks), K), dtype=np.float16)
    X[np.arange(len(ks)), ks] = 1.0
    Y = orc.linear(X, q, s)
    for m, k in enumerate(ks):
        assert np.array_equal(Y[m], q[k].astype(np.float64) * s.astype(np.float64))


def pin_linear_against_exact_rationals(orc):
    X = synthetic.activations(2, 5, SEED, 91)
    q = np.array([[3, -127, 0], [127, 5, -6], [-1, 2, 99], [64, -64, 1], [0, 0, -7]], dtype=np.int8)
    s = np.array([0.001, 0.0625, 3.5e-4], dtype=np.float16)
    b = np.array([0.5, -0.25, 0.0], dtype=np.float16)
    Y = orc.linear(X, q, s, b)
    for m in range(2):
        for n in range(3):
            acc = sum(Fraction(float(X[m, k])) * int(q[k, n]) for k in range(5))
            exact = acc * Fraction(float(s[n])) + Fraction(float(b[n]))
            assert abs(Fraction(Y[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 50)


def pin_linear_matches_numpy_matmul(orc):
    M, K, N = 4, 256, 512
    W = synthetic.weights(K, N, SEED, 101)
    X = synthetic.activations(M, K, SEED, 102)
    b = synthetic.bias(N, SEED, 103)
    q, s = orc.quantize(W)
    Y = orc.linear(X, q, s, b)
    ref = X.astype(np.float64) @ (q.astype(np.float64) * s.astype(np.float64)) + b.astype(np.float64)
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)


def pin_cosine_similarity_as_printed(orc):
    g = golden.load("w8a16_cosine.txt")
    K, N, M = 4096, 256, 4
    W = synthetic.weights(K, N, SEED, 111, outlier_frac=0.001)
    X = synthetic.activations(M, K, SEED, 112)
    q, s = orc.quantize(W)
    Yq = orc.linear(X, q, s).ravel()
    Yf = (X.astype(np.float64) @ W.astype(np.float64)).ravel()
    cos = float(Yq @ Yf / (np.linalg.norm(Yq) * np.linalg.norm(Yf)))
    assert cos > g["min_cosine"]


def pin_tolerance_helper_rejects_a_planted_error(orc):
    M, K, N = 4, 256, 512
    q, s = orc.quantize(synthetic.weights(K, N, SEED, 121))
    X = synthetic.activations(M, K, SEED, 122)
    Y = orc.linear(X, q, s)
    Y16 = Y.astype(np.float16).astype(np.float64)
    assert oracle.tolerance_ok(Y16, Y)[0]
    bad = Y16.copy()
    bad[1, 7] += 4e-3 * np.abs(Y).max()
    assert not oracle.tolerance_ok(bad, Y)[0]
    # a dropped scale on one channel is caught
    s_bad = s.copy()
    s_bad[3] = np.float16(float(s[3]) * 1.01)
    assert not oracle.tolerance_ok(orc.linear(X, q, s_bad), Y)[0]


# ---------------------------------------------------------------- asymmetric (affine) quantization
# (q - z) S with S = (hi - lo) / 255 over a range that includes 0 and
# z = rne(-128 - lo / S): pinned to values fixed by construction.

def pin_asym_integer_grid_round_trips(orc):
    # W = (i - z) S exactly, with i spanning -128..127 in every column: the
    # range is exactly 255 S, so the scale, the zero point and every code
    # come back unchanged
    rng = np.random.default_rng(41)
    K, N = 300, 24
    S = np.array([2.0 ** -e * (1 + f / 1024) for e, f in zip(rng.integers(3, 12, N), rng.integers(0, 1024, N))],
                 dtype=np.float16)
    Z = rng.integers(-128, 128, N).astype(np.int32)
    I = rng.integers(-128, 128, size=(K, N)).astype(np.int32)
    I[0] = -128
    I[1] = 127
    W = ((I - Z) * S.astype(np.float64)).astype(np.float32)
    assert np.array_equal(W.astype(np.float64), (I - Z) * S.astype(np.float64))   # exact in fp32
    q, s, z = orc.quantize_asym(W)
    assert np.array_equal(s.view(np.uint16), S.view(np.uint16))
    assert np.array_equal(z.astype(np.int32), Z)
    assert np.array_equal(q.astype(np.int32), I)


def pin_asym_zero_weight_is_exact_and_sign_ranges(orc):
    rng = np.random.default_rng(42)
    K = 257
    pos = np.abs(rng.standard_normal(K)).astype(np.float32)
    neg = -np.abs(rng.standard_normal(K)).astype(np.float32)
    mixed = rng.standard_normal(K).astype(np.float32)
    W = np.stack([pos, neg, mixed], axis=1)
    W[5] = 0.0
    q, s, z = orc.quantize_asym(W)
    # 0 is always representable: a zero weight is stored as the zero point
    assert np.array_equal(q[5], z)
    # all weights >= 0: the range starts at 0, z = -128, the largest is 127
    assert z[0] == -128 and q[np.argmax(pos), 0] == 127 and q[:, 0].min() >= -128
    # all weights <= 0: the range ends at 0, z = 127, the smallest is -128
    assert z[1] == 127 and q[np.argmin(neg), 1] == -128
    # mixed signs: the extremes map to the ends of the code range
    assert q[np.argmin(mixed), 2] == -128 and q[np.argmax(mixed), 2] == 127
    # strictly positive weights far from 0: the range still starts at 0, so
    # the smallest weight is NOT on the bottom level
    lifted = (np.abs(rng.standard_normal((K, 2))) + 1.0).astype(np.float32)
    ql, sl, zl = orc.quantize_asym(lifted)
    assert np.all(zl == -128)
    # with lo = 0 the scale is the symmetric bound's formula over 255 levels
    top = lifted.max(axis=0)
    assert np.array_equal(sl, (top / np.float32(255.0)).astype(np.float16))
    assert np.all(ql.min(axis=0) > -128 + 50)
    # an all-zero column: scale 0, zero point 0, codes 0
    q0, s0, z0 = orc.quantize_asym(np.zeros((16, 8), dtype=np.float32))
    assert not q0.any() and not s0.view(np.uint16).any() and not z0.any()


def pin_asym_divides_by_the_stored_fp16_scale(orc):
    # As for the symmetric codes, the weights are divided by the scale that
    # is stored (fp16), not by the fp32 range / 255 it was rounded from.  A
    # column over [0, 1] has z = -128 and S = fp16(1/255) != 1/255; one
    # weight sits where the two scales give different codes.
    hi = np.float32(1.0)
    s32 = hi / np.float32(255.0)
    s16 = np.float32(np.float16(s32))
    assert s16 != s32
    # the two scales differ by about 1.5e-5 relatively, so the weight sits
    # high in the range and within a few thousandths of a half-integer
    w = by16 = by32 = None
    for x in (np.float32(200.501), np.float32(200.499), np.float32(240.5015), np.float32(240.4985)):
        w = x * s16
        by16, by32 = np.rint(w / s16), np.rint(w / s32)
        if by16 != by32:
            break
    assert by16 != by32                         # the case distinguishes them
    q, s, z = orc.quantize_asym(np.array([[0.0], [hi], [w]], dtype=np.float32))
    assert np.float32(s[0]) == s16 and z[0] == -128
    assert q[1, 0] == 127 and q[0, 0] == -128
    assert int(q[2, 0]) == int(by16) - 128


def pin_asym_reconstruction_error_bound(orc):
    # |w - (q - z) S| <= S / 2, widened by the scale's fp16 rounding, which
    # can stretch the top of the range by up to 255 * 2^-11 of a level
    K, N = 512, 96
    W = synthetic.weights(K, N, SEED, 131, outlier_frac=0.01)
    W[:, :8] = np.abs(W[:, :8])
    for Wt in (W, W.astype(np.float16)):
        q, s, z = orc.quantize_asym(Wt)
        sf = s.astype(np.float64)
        deq = (q.astype(np.float64) - z.astype(np.float64)) * sf
        err = np.abs(deq - Wt.astype(np.float64))
        assert np.all(err <= (0.5 + 255 * 2.0 ** -11 + 2.0 ** -10) * sf + 1e-12)
        # the column extremes land within one level of the ends of the code
        # range (the rounding of S and of z may each move them by a fraction)
        assert np.all(q.min(axis=0) <= -127) and np.all(q.max(axis=0) >= 126)


def pin_asym_linear_unit_rows_and_reductions(orc):
    rng = np.random.default_rng(43)
    K, N = 64, 40
    q = rng.integers(-128, 128, size=(K, N)).astype(np.int8)
    s = (rng.uniform(0.5, 2.0, N) / 64).astype(np.float16)
    z = rng.integers(-128, 128, N).astype(np.int8)
    b = (rng.integers(-64, 64, N) / 8).astype(np.float16)
    # unit rows pick one dequantized weight row: (q[k] - z) S + bias, exactly
    ks = [0, 17, 63]
    X = np.zeros((len(ks), K), dtype=np.float16)
    X[np.arange(len(ks)), ks] = 1.0
    Y = orc.linear_asym(X, q, s, z, b)
    want = (q[ks].astype(np.float64) - z.astype(np.float64)) * s.astype(np.float64) + b.astype(np.float64)
    assert np.array_equal(Y, want)
    # a zero point of 0 is the symmetric product
    Xr = synthetic.activations(5, K, SEED, 132)
    assert np.array_equal(orc.linear_asym(Xr, q, s, np.zeros(N, np.int8), b), orc.linear(Xr, q, s, b))
    # shifting every code and its zero point by the same amount changes nothing
    q2 = np.clip(q.astype(np.int32), -120, 120)
    z2 = np.clip(z.astype(np.int32), -120, 120)
    Y1 = orc.linear_asym(Xr, q2.astype(np.int8), s, z2.astype(np.int8))
    Y2 = orc.linear_asym(Xr, (q2 + 7).astype(np.int8), s, (z2 + 7).astype(np.int8))
    assert np.allclose(Y1, Y2, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- clipped scale
# bound = min(max|W|, c) or the ceil(pK)-th smallest |W| per channel, then
# the symmetric quantizer: pinned to order statistics known by construction.

def pin_clip_reduces_to_symmetric(orc):
    W = synthetic.weights(300, 48, SEED, 141, outlier_frac=0.01)
    q, s = orc.quantize(W)
    for mode, param in (("percentile", 1.0), ("fixed", float("inf")), ("fixed", 1e30)):
        qc, sc = orc.quantize_clip(W, mode, param)
        assert np.array_equal(qc, q) and np.array_equal(sc.view(np.uint16), s.view(np.uint16))


def pin_percentile_bound_is_the_order_statistic(orc):
    # each column holds |w| = delta, 2 delta, ..., K delta (shuffled, random
    # signs): the r-th smallest magnitude is r delta exactly
    rng = np.random.default_rng(44)
    K, N, delta = 400, 12, 2.0 ** -10
    W = np.empty((K, N), dtype=np.float32)
    for n in range(N):
        W[:, n] = rng.permutation(np.arange(1, K + 1)) * delta * rng.choice([-1.0, 1.0], K)
    for p, r in ((0.9501, 381), (0.5, 200), (0.999, 400), (0.0001, 1), (0.75, 300)):
        q, s = orc.quantize_clip(W, "percentile", p)
        want = np.float16(np.float32(r * delta) / np.float32(127.0))
        assert np.all(s == want), (p, r)
        # everything at or beyond the bound is clipped onto +-127, nothing
        # well below it is
        mag = np.abs(W)
        assert np.all(np.abs(q[mag >= r * delta]) == 127), (p, r)
        assert np.all(np.abs(q[mag < 0.99 * r * delta]) < 127), (p, r)


def pin_percentile_monotone_in_p(orc):
    W = synthetic.weights(512, 40, SEED, 142, outlier_frac=0.01)
    prev = None
    for p in (0.5, 0.9, 0.99, 0.999, 1.0):
        _, s = orc.quantize_clip(W, "percentile", p)
        sf = s.astype(np.float64)
        if prev is not None:
            assert np.all(sf >= prev)
        prev = sf


def pin_fixed_clip_scale_and_codes(orc):
    W = synthetic.weights(256, 32, SEED, 143, outlier_frac=0.01)
    c = 127.0 * 2.0 ** -12         # below every column's max: S = 2^-12 exactly
    assert np.all(np.abs(W).max(axis=0) > c)
    q, s = orc.quantize_clip(W, "fixed", c)
    assert np.all(s == np.float16(2.0 ** -12))
    inside = np.abs(W) <= c
    err = np.abs(q.astype(np.float64) * 2.0 ** -12 - W.astype(np.float64))
    assert np.all(err[inside] <= 2.0 ** -13)
    assert np.all(np.abs(q[np.abs(W) >= c * (1 + 2 ** -7)]) == 127)
    # a clip above a column's max leaves that column unclipped
    W2 = W.copy()
    W2[:, 5] *= 0.1
    q2, s2 = orc.quantize_clip(W2, "fixed", c)
    qs, ss = orc.quantize(W2[:, 5:6])
    assert s2[5] == ss[0] and np.array_equal(q2[:, 5], qs[:, 0])


def pin_fixed_clip_param_is_an_fp32_value(orc):
    # The C ABI passes the clip as a double but defines the bound in fp32:
    # bound = min(max|W|, c) with c = fp32(clip_param).  For fp32 weights a
    # comparison made in double selects the same bound (no fp32 value lies
    # strictly between c and fp32(c) on the side that would differ), so what
    # is pinned is the value the bound takes.  The c used is not an fp32
    # value; fp32(c) lies just above it, and it is chosen where fp32(c)/127
    # and the quotient of the fp32 value below fp32(c) round to different
    # fp16 scales, so a bound that is off by one fp32 step changes the
    # scale.  A column whose max is exactly fp32(c) lies between c and
    # fp32(c): it is not clipped.  Clipping a column then equals the plain
    # quantizer (pinned above) on the same column with its entries clamped
    # to +-fp32(c).
    c = 0.0900199469178915
    c32 = np.float32(c)
    assert float(c32) != c and float(c32) > c
    below = np.nextafter(c32, np.float32(0))
    assert np.float16(c32 / np.float32(127)) != np.float16(below / np.float32(127))
    W = synthetic.weights(300, 24, SEED, 147, outlier_frac=0.02) * np.float32(4.0)
    W[7, 3] = c32                       # column 3: max exactly fp32(c)
    W[:, 3] = np.clip(W[:, 3], -c32, c32)
    W[:, 9] = np.clip(W[:, 9], -c32, c32) * np.float32(0.5)   # column 9: below c
    q, s = orc.quantize_clip(W, "fixed", c)
    q32, s32 = orc.quantize_clip(W, "fixed", float(c32))
    assert np.array_equal(q, q32) and np.array_equal(s.view(np.uint16), s32.view(np.uint16))
    qc, sc = orc.quantize(np.clip(W, -c32, c32))
    assert np.array_equal(q, qc) and np.array_equal(s.view(np.uint16), sc.view(np.uint16))
    q3, s3 = orc.quantize(np.ascontiguousarray(W[:, 3:4]))
    assert s[3] == s3[0] and np.array_equal(q[:, 3], q3[:, 0])
    assert np.sum(np.abs(W).max(axis=0) > c32) >= 20      # most columns are clipped


# ---------------------------------------------------------------- outlier split
# weights above the percentage-clip bound kept apart as fp16, code 0; the
# rest quantized with that bound.

def pin_outliers_p_one_is_the_symmetric_quantizer(orc):
    W = synthetic.weights(300, 40, SEED, 151, outlier_frac=0.01)
    q, s, cnt, rows, vals = orc.quantize_outliers(W, 1.0)
    q0, s0 = orc.quantize(W)
    assert rows.shape == (40, 0) and not cnt.any()
    assert np.array_equal(q, q0) and np.array_equal(s.view(np.uint16), s0.view(np.uint16))
    X = synthetic.activations(3, 300, SEED, 152)
    assert np.array_equal(orc.linear_outliers(X, q, s, cnt, rows, vals), orc.linear(X, q0, s0))


def pin_outliers_are_the_largest_magnitudes(orc):
    # |w| = delta, 2 delta, ..., K delta per column (shuffled, random signs):
    # the outliers are exactly the K - r largest, in increasing row order
    rng = np.random.default_rng(45)
    K, N, delta = 400, 10, 2.0 ** -10
    W = np.empty((K, N), dtype=np.float32)
    for n in range(N):
        W[:, n] = rng.permutation(np.arange(1, K + 1)) * delta * rng.choice([-1.0, 1.0], K)
    for p, r in ((0.99, 396), (0.9501, 381)):
        q, s, cnt, rows, vals = orc.quantize_outliers(W, p)
        cap = K - r
        assert rows.shape == (N, cap) and np.all(cnt == cap)
        for n in range(N):
            want = np.sort(np.argsort(np.abs(W[:, n]))[r:])
            assert np.array_equal(rows[n], want)
            assert np.array_equal(vals[n].astype(np.float32), W[want, n])   # exact in fp16
            assert not q[want, n].any()
        assert np.all(s == np.float16(np.float32(r * delta) / np.float32(127.0)))


def pin_outlier_split_reconstructs_the_weight(orc):
    K, N = 512, 64
    W = synthetic.weights(K, N, SEED, 153, outlier_frac=0.01)
    for p in (0.999, 0.99, 0.95):
        q, s, cnt, rows, vals = orc.quantize_outliers(W, p)
        deq = q.astype(np.float64) * s.astype(np.float64)
        for n in range(N):
            deq[rows[n, :cnt[n]], n] += vals[n, :cnt[n]].astype(np.float64)
            assert np.all(np.diff(rows[n, :cnt[n]]) > 0) and not rows[n, cnt[n]:].any()
        is_out = np.zeros((K, N), dtype=bool)
        for n in range(N):
            is_out[rows[n, :cnt[n]], n] = True
        err = np.abs(deq - W.astype(np.float64))
        sf = s.astype(np.float64)
        assert np.all(err[~is_out] <= (0.5 + 2.0 ** -10) * np.broadcast_to(sf, (K, N))[~is_out])
        assert np.all(err[is_out] <= 2.0 ** -11 * np.abs(W.astype(np.float64))[is_out])


def pin_outlier_linear_unit_rows(orc):
    K, N = 200, 24
    W = synthetic.weights(K, N, SEED, 154, outlier_frac=0.02)
    q, s, cnt, rows, vals = orc.quantize_outliers(W, 0.97)
    b = synthetic.bias(N, SEED, 155)
    ks = [int(rows[0, 0]), 5, 199]
    X = np.zeros((len(ks), K), dtype=np.float16)
    X[np.arange(len(ks)), ks] = 1.0
    Y = orc.linear_outliers(X, q, s, cnt, rows, vals, b)
    for i, k in enumerate(ks):
        want = q[k].astype(np.float64) * s.astype(np.float64) + b.astype(np.float64)
        for n in range(N):
            hit = np.nonzero(rows[n, :cnt[n]] == k)[0]
            if hit.size:
                want[n] += float(vals[n, hit[0]])
        assert np.array_equal(Y[i], want)


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__[4:] for p in PINS])
def test_oracle_pin(pin):
    pin(oracle.default())
