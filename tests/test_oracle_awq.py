"""Pins of the oracle's awq_w4a16 step ("Nunchaku Lite in Diffusers": int4 weights in groups of
64 with 16-bit activations, for the modulation projections) to exact constructions, the
rounding rule's error bound, ties, special cases and brute-force dot products."""
import numpy as np
import pytest

from oracle import svdq_oracle as O


def _grid_group(rng, s, z):
    q = rng.integers(0, 16, 64)
    q[rng.integers(0, 64)] = 0
    q[rng.integers(0, 64)] = 15
    q[0], q[1] = 0, 15
    return q, (q - z) * s


@pytest.mark.parametrize("s,z", [(2.0 ** -7, 5), (2.0 ** -3, 0), (2.0 ** -10, 15), (0.375, 8)])
def test_representable_groups_are_lossless(s, z):
    rng = np.random.default_rng(1)
    rows = [_grid_group(rng, s, z) for _ in range(3)]
    W = np.stack([np.concatenate([w, w[::-1]]) for _, w in rows]).astype(np.float32)
    q, sc, zz = O.awq_quantize(W)
    assert np.all(sc == s) and np.all(zz == z)
    np.testing.assert_array_equal(O.awq_dequantize(q, sc, zz), W.astype(np.float64))


def test_round_to_nearest_error_bound_and_monotone():
    rng = np.random.default_rng(2)
    W = rng.normal(0, 0.02, (16, 256)).astype(np.float32)
    W[3, :64] += 0.5  # a group far from zero (zero point clamps at 0)
    q, s, z = O.awq_quantize(W)
    Wh = O.awq_dequantize(q, s, z)
    sg = np.repeat(s, 64, axis=1)
    inner = (q > 0) & (q < 15)
    err = np.abs(W.astype(np.float64) - Wh)
    assert np.all(err[inner] <= 0.5 * sg[inner] * (1 + 2.0 ** -20) + np.abs(W[inner]) * 2.0 ** -23)
    # groups whose range holds zero (z not clamped): every element within 1.5 steps
    G = W.reshape(16, 4, 64)
    straddle = np.repeat((G.min(axis=2) <= 0) & (G.max(axis=2) >= 0), 64, axis=1)
    assert np.all(err[straddle] <= 1.5 * sg[straddle])
    # the shifted group: -min / s < 0 clamps z at 0, the grid [0, 15 s] lies below the values
    # and every code saturates at 15 (the zero-point clamp of the storage format)
    assert z[3, 0] == 0 and np.all(q[3, :64] == 15)
    for n in range(W.shape[0]):
        for g in range(W.shape[1] // 64):
            w = W[n, 64 * g:64 * g + 64]
            o = np.argsort(w, kind="stable")
            assert np.all(np.diff(q[n, 64 * g:64 * g + 64][o].astype(int)) >= 0)


def test_ties_round_to_even():
    s = 2.0 ** -6
    # grid offsets k + 1/2 for k = -8 .. 6 (plus the extremes that fix z = 8, s = 2^-6)
    w = np.array([-8.0, 7.0] + [k + 0.5 for k in range(-8, 7)] * 4 + [0.0] * 2) * s
    W = w[None, :64].astype(np.float32)
    q, sc, zz = O.awq_quantize(W)
    assert sc[0, 0] == s and zz[0, 0] == 8
    d = q[0].astype(int) - 8
    halves = np.abs(W[0] / s - np.floor(W[0] / s) - 0.5) < 1e-12
    assert np.all(d[halves] % 2 == 0)
    np.testing.assert_array_equal(d[halves], np.rint(W[0][halves] / s).astype(int))


def test_zero_and_constant_groups():
    W = np.zeros((2, 128), np.float32)
    W[1, 64:] = 0.25
    q, s, z = O.awq_quantize(W)
    # range below 1e-5 takes 1e-5: s = fp16(fp32(1e-5 / 15))
    assert s[0, 0] == float(np.float16(np.float32(np.float32(1e-5) / np.float32(15.0))))
    assert np.all(O.awq_dequantize(q, s, z)[0] == 0.0)
    # a positive constant group: z = 0 and the codes saturate at 15
    assert z[1, 1] == 0 and np.all(q[1, 64:] == 15)


def test_linear_brute_force():
    rng = np.random.default_rng(3)
    N, K, M = 24, 192, 3
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    X = rng.normal(size=(M, K))
    b = rng.normal(0, 0.01, N)
    q, s, z = O.awq_quantize(W)
    Y = O.awq_linear(X, q, s, z, b)
    for m, n in [(0, 0), (2, 23), (1, 7), (0, 13)]:
        acc = 0.0
        for k in range(K):
            g = k // 64
            acc += (int(q[n, k]) - int(z[n, g])) * s[n, g] * X[m, k]
        assert abs(Y[m, n] - (acc + b[n])) <= 1e-12 * (1 + abs(acc))


def test_pins_catch_planted_mistakes():
    rng = np.random.default_rng(4)
    q0, w = _grid_group(rng, 2.0 ** -7, 5)
    W = w[None, :].astype(np.float32)
    q, s, z = O.awq_quantize(W)
    good = O.awq_dequantize(q, s, z)
    # zero point added instead of subtracted; scale taken per 32 instead of 64; no zero point
    bad1 = (q.astype(float) + z[0, 0]) * s[0, 0]
    bad2 = O.awq_dequantize(*O.awq_quantize(W, group=32), group=32)
    bad3 = q.astype(float) * s[0, 0]
    for bad in (bad1, bad3):
        assert not np.array_equal(bad, W.astype(np.float64))
    assert np.array_equal(good, W.astype(np.float64))
    assert bad2.shape == good.shape

