"""Pins of the fp64 oracle to things other than itself.

Each test ties one step of the oracle to the format definitions, a closed form, an
invariant of the method, a library special case or a brute-force recomputation, so
that a dropped term, a wrong sign or index or a transposed operand fails somewhere.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import svdq_oracle as O
from synth import CONFIGS, bf16_bits_to_f32, f32_to_bf16_bits, make_inputs
from tests import svdq_formats as F

HERE = os.path.dirname(os.path.abspath(__file__))


# ------------------------------------------------------------------ formats
def test_e2m1_table_matches_format_definition():
    np.testing.assert_array_equal(F.e2m1_table(), O.E2M1_MAGNITUDES)


def test_e2m1_codes_round_trip():
    for c in range(16):
        if c == 8:  # -0 is not produced: zero encodes as +0
            continue
        v = O.e2m1_decode(np.array([c], np.uint8))
        assert O.e2m1_encode(O.e2m1_round(v))[0] == c


@pytest.mark.parametrize(
    "x,want",
    [(0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0), (3.5, 4.0), (5.0, 4.0),
     (6.0, 6.0), (7.0, 6.0), (1e9, 6.0), (-0.25, 0.0), (-0.75, -1.0), (-5.0, -4.0), (-100.0, -6.0),
     (0.2499999, 0.0), (0.2500001, 0.5), (4.9999, 4.0), (5.0001, 6.0)],
)
def test_e2m1_ties_and_saturation(x, want):
    assert O.e2m1_round(np.array([x]))[0] == want
    assert F.brute_e2m1(x) == want


def test_e2m1_negative_zero_encodes_positive():
    assert O.e2m1_encode(O.e2m1_round(np.array([-0.1, -0.0])))[0] == 0
    assert O.e2m1_encode(O.e2m1_round(np.array([-0.0])))[0] == 0


def test_e2m1_matches_brute_force_table_search():
    rng = np.random.default_rng(1)
    xs = np.concatenate([rng.uniform(-8, 8, 3000), np.arange(-8, 8.001, 0.125)])
    xs = O.f32(xs)
    got = O.e2m1_round(xs)
    want = np.array([F.brute_e2m1(x) for x in xs])
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(O.e2m1_encode(got), [F.brute_e2m1_code(x) for x in xs])


def test_e4m3_table_and_codes():
    t = F.e4m3_table()
    assert t[0x7E] == 448.0 and t[0x01] == 2.0 ** -9 and t[0x08] == 2.0 ** -6
    codes = np.arange(0x7F, dtype=np.uint8)
    np.testing.assert_array_equal(O.e4m3_decode(codes), t)
    np.testing.assert_array_equal(O.e4m3_encode(t), codes)
    np.testing.assert_array_equal(O.e4m3_round(t), t)


def test_e4m3_matches_brute_force_table_search():
    rng = np.random.default_rng(2)
    t = F.e4m3_table()
    mids = (t[1:] + t[:-1]) / 2  # every tie
    xs = np.concatenate([
        np.exp(rng.uniform(np.log(2.0 ** -12), np.log(600.0), 4000)),
        mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
        [0.0, 2.0 ** -10, 2.0 ** -10 * 1.0001, 448.0, 449.0, 464.0, 479.9, 480.0, 1e6],
    ])
    xs = O.f32(xs)
    got = O.e4m3_round(xs)
    want = np.array([F.brute_e4m3(x) for x in xs])
    np.testing.assert_array_equal(got, want)


def test_bf16_round_matches_integer_rounding():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    via_bits = bf16_bits_to_f32(f32_to_bf16_bits(x)).astype(np.float64)
    np.testing.assert_array_equal(O.bf16_round(x.astype(np.float64)), via_bits)


def test_pack_nibble_order():
    codes = np.array([[1, 2, 3, 4, 0xF, 0]], np.uint8)
    packed = O.pack_codes(codes)
    np.testing.assert_array_equal(packed, [[0x21, 0x43, 0x0F]])
    np.testing.assert_array_equal(O.unpack_codes(packed), codes)


# ------------------------------------------------------------------ NVFP4
def _brute_group(v, s):
    """Scalar restatement of the group quantizer with table-search rounding."""
    amax = max(abs(x) for x in v)
    d = float(np.float32(6.0 * s))
    sg = F.brute_e4m3(float(np.float32(amax / d)))
    if sg == 0.0:
        return [0] * 16, sg
    eff = float(np.float32(sg * s))
    return [F.brute_e2m1_code(float(np.float32(x / eff))) for x in v], sg


def test_nvfp4_group_matches_scalar_restatement():
    rng = np.random.default_rng(4)
    rows = O.f32(rng.standard_normal((6, 64)) * np.exp(rng.uniform(-3, 3, (6, 1))))
    rows[2, 16:32] = 0.0
    rows[3, :16] *= 1e-6  # a group whose scale underflows to zero
    s = O.tensor_scale(np.abs(rows).max())
    codes, scales = O.nvfp4_quantize(rows, s)
    for i in range(rows.shape[0]):
        for g in range(4):
            c, sg = _brute_group(rows[i, 16 * g:16 * g + 16], s)
            assert list(codes[i, 16 * g:16 * g + 16]) == c
            assert O.e4m3_decode(scales[i, g]) == sg


@pytest.mark.parametrize("k", [-9, -3, 0, 2, 8])
def test_nvfp4_lossless_on_grid_values(k):
    # amax = 6 * 2^k with s = 1: the group scale is 2^k (exact in e4m3) and every
    # element divided by it is an e2m1 value, so dequantization returns the input.
    rng = np.random.default_rng(10 + k)
    grid = np.concatenate([O.E2M1_MAGNITUDES, -O.E2M1_MAGNITUDES[1:]])
    v = rng.choice(grid, (3, 32))
    v[:, 0] = 6.0
    v[:, 16] = -6.0
    v = v * 2.0 ** k
    codes, scales = O.nvfp4_quantize(v, 1.0)
    np.testing.assert_array_equal(O.e4m3_decode(scales), 2.0 ** k)
    np.testing.assert_array_equal(O.nvfp4_dequantize(codes, scales), v)


def test_nvfp4_error_bound():
    # Without saturation each element is off by at most half an e2m1 step times its
    # effective scale: <= 1 * eff (the 4..6 interval) and <= 0.25 * eff below 2.
    rng = np.random.default_rng(5)
    v = O.f32(rng.standard_normal((50, 256)))
    s = O.tensor_scale(np.abs(v).max())
    codes, scales = O.nvfp4_quantize(v, s)
    deq = O.nvfp4_dequantize(codes, scales) * s
    eff = (O.e4m3_decode(scales) * s).repeat(16, axis=1)
    err = np.abs(deq - v)
    q = np.abs(v) / eff
    sat = q > 6.0
    bound = np.where(q < 2, 0.25, np.where(q < 4, 0.5, 1.0)) * eff * (1 + 1e-6)
    assert np.all(err[~sat] <= bound[~sat])
    assert np.all(np.abs(deq[sat]) == 6.0 * eff[sat])


# -------------------------------------------------------------- smoothing
def test_smoothing_closed_form():
    lam, inv = O.smoothing_factors(np.array([4.0, 9.0, 0.0, 1.0]), np.array([0.25, 0.04, 1.0, 0.0]))
    np.testing.assert_array_equal(lam, [4.0, 15.0, 1.0, 1.0])
    np.testing.assert_array_equal(inv, O.f32([0.25, 1 / 15.0, 1.0, 1.0]))


def test_smoothing_balances_channel_maxima():
    # With exponent 1/2 the smoothed activation and weight maxima meet at sqrt(a_x a_w).
    Xb, W, b, ch = make_inputs(CONFIGS["tiny"])
    X = bf16_bits_to_f32(Xb).astype(np.float64)
    a_x = O.calibration_absmax(X)
    a_w = np.abs(W.astype(np.float64)).max(axis=0)
    lam, inv = O.smoothing_factors(a_x, a_w)
    target = np.sqrt(a_x * a_w)
    np.testing.assert_allclose(a_x * inv, target, rtol=1e-6)
    np.testing.assert_allclose(a_w * lam, target, rtol=1e-6)
    # outlier channels get the largest factors
    assert set(np.argsort(lam)[-4:]) == set(ch)


# --------------------------------------------------------------------- SVD
def _known_svd(K, N, p, seed=6):
    rng = np.random.default_rng(seed)
    U, _ = np.linalg.qr(rng.standard_normal((K, p)))
    V, _ = np.linalg.qr(rng.standard_normal((N, p)))
    s = np.sort(rng.uniform(1, 10, p))[::-1] + np.arange(p)[::-1] * 0.5
    return U, s, V, (U * s) @ V.T


def test_svd_split_recovers_constructed_singular_values():
    U, s, V, A = _known_svd(48, 40, 12)
    P, sig, Q = O.svd_split(A, 12)
    np.testing.assert_allclose(sig, s, rtol=1e-12)
    np.testing.assert_allclose(P.T @ P, np.eye(12), atol=1e-12)
    np.testing.assert_allclose((P * sig) @ Q.T, A, atol=1e-11)
    # same subspace, up to the sign convention
    np.testing.assert_allclose(np.abs(np.sum(P * U, axis=0)), 1.0, atol=1e-10)
    idx = np.argmax(np.abs(P), axis=0)
    assert np.all(P[idx, np.arange(12)] > 0)


def test_svd_split_truncation_is_best_rank_r():
    # Eckart-Young: the rank-r error in Frobenius norm is the root sum of the dropped sigma^2.
    U, s, V, A = _known_svd(30, 50, 20, seed=7)
    P, sig, Q = O.svd_split(A, 8)
    err = np.linalg.norm(A - (P * sig) @ Q.T)
    np.testing.assert_allclose(err, math.sqrt(np.sum(s[8:] ** 2)), rtol=1e-10)


# ----------------------------------------------------------- layer invariants
def _tiny_problem(M=64, K=128, N=96, seed=8):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    X[:, [3, K - 5]] *= 30
    X = bf16_bits_to_f32(f32_to_bf16_bits(X.astype(np.float32))).astype(np.float64)
    W = O.f32(rng.normal(0, 0.02, (N, K)))
    W[:, [3, K - 5]] *= 0.2
    W = O.f32(W)
    b = O.f32(rng.normal(0, 0.01, N))
    return X, W, b


def test_full_rank_branch_reproduces_dense_layer():
    X, W, b = _tiny_problem()
    r = min(W.shape)
    layer = O.prepare(W, b, O.calibration_absmax(X), r, branch="fp64")
    assert np.abs(layer.R).max() < 1e-13 * np.abs(W).max() * layer.lam.max()
    Y = O.layer_forward(X, layer)
    Y_dense = X @ W.T + b
    assert np.abs(Y - Y_dense).max() <= 1e-10 * np.abs(Y_dense).max()


def test_full_rank_bf16_branch_error_is_bf16_level():
    X, W, b = _tiny_problem()
    layer = O.prepare(W, b, O.calibration_absmax(X), min(W.shape), branch="bf16")
    Y = O.layer_forward(X, layer)
    Y_dense = X @ W.T + b
    rel = np.linalg.norm(Y - Y_dense) / np.linalg.norm(Y_dense)
    assert rel < 2e-2


def _brute_w4a4(X, W, b):
    """Plain W4A4 (no smoothing, no branch) by scalar loops over table-rounded values."""
    def q_rows(A):
        s = float(np.float32(np.abs(A).max() / 2688.0))
        out = np.zeros_like(A)
        for i in range(A.shape[0]):
            for g in range(A.shape[1] // 16):
                v = A[i, 16 * g:16 * g + 16]
                codes, sg = _brute_group(v, s)
                for j, c in enumerate(codes):
                    mag = F.e2m1_table()[c & 7]
                    out[i, 16 * g + j] = (-mag if c & 8 else mag) * sg
        return out, s

    Xq, sx = q_rows(X)
    Wq, sw = q_rows(W)
    Y = np.zeros((X.shape[0], W.shape[0]))
    for m in range(X.shape[0]):
        for n in range(W.shape[0]):
            acc = 0.0
            for k in range(X.shape[1]):
                acc += Xq[m, k] * Wq[n, k]
            Y[m, n] = sx * sw * acc + b[n]
    return Y


def test_rank_zero_unit_lambda_is_plain_w4a4():
    X, W, b = _tiny_problem(M=8, K=64, N=12)
    layer = O.prepare(W, b, O.calibration_absmax(X), 0, unit_lambda=True)
    Y = O.layer_forward(X, layer)
    np.testing.assert_allclose(Y, _brute_w4a4(X, W, b), rtol=1e-12, atol=1e-12)


def test_brute_force_dot_products():
    X, W, b = _tiny_problem()
    layer = O.prepare(W, b, O.calibration_absmax(X), 16)
    xc, xs, La = O.quant_act_lora_down(X, layer)
    Y = O.gemm_w4a4_lora_up(xc, xs, La, layer)
    rng = np.random.default_rng(9)
    for m, n in zip(rng.integers(0, X.shape[0], 20), rng.integers(0, W.shape[0], 20)):
        acc = 0.0
        for k in range(X.shape[1]):
            xv = O.E2M1_MAGNITUDES[xc[m, k] & 7] * (-1 if xc[m, k] & 8 else 1) * O.e4m3_decode(xs[m, k // 16])
            wv = O.E2M1_MAGNITUDES[layer.w_codes[n, k] & 7] * (-1 if layer.w_codes[n, k] & 8 else 1) \
                * O.e4m3_decode(layer.w_scales[n, k // 16])
            acc += xv * wv
        lora = 0.0
        for j in range(layer.rank):
            xb = 0.0
            for k in range(X.shape[1]):
                xb += X[m, k] * layer.L1[k, j]
            lora += xb * layer.L2[j, n]
        want = layer.s_x * layer.s_w * acc + lora + b[n]
        assert abs(Y[m, n] - want) <= 1e-12 * max(1.0, abs(want))


def test_low_rank_branch_absorbs_outliers():
    # The method's claim: with outliers in X, the low-rank branch lowers the 4-bit error.
    Xb, W, b, _ = make_inputs(CONFIGS["tiny"])
    X = bf16_bits_to_f32(Xb).astype(np.float64)
    Y_dense = X @ W.astype(np.float64).T + b
    a_x = O.calibration_absmax(X)

    def err(rank, unit_lambda=False):
        layer = O.prepare(W, b, a_x, rank, unit_lambda=unit_lambda)
        return np.linalg.norm(O.layer_forward(X, layer) - Y_dense) / np.linalg.norm(Y_dense)

    e_plain, e_smooth, e_r16, e_r64 = err(0, True), err(0), err(16), err(64)
    assert e_r64 < e_r16 < e_smooth < e_plain


def test_folded_branch_equals_smoothed_input_branch():
    # Unrounded branch: X L1s equals X_hat (P_r S_r^1/2), the down-projection of the smoothed
    # input, with P, S from an SVD of W_hat^T taken here (the factor's sign choice cancels in
    # the projector P_r P_r^T, so compare the rank-r products against L2).
    X, W, b = _tiny_problem()
    r = 8
    layer = O.prepare(W, b, O.calibration_absmax(X), r, branch="fp64")
    Xh = X / layer.lam[None, :]
    U, S, Vh = np.linalg.svd((W * layer.lam[None, :]).T, full_matrices=False)
    want = Xh @ U[:, :r] @ np.diag(S[:r]) @ Vh[:r]
    got = (X @ layer.L1) @ layer.L2
    assert np.abs(got - want).max() <= 1e-10 * np.abs(want).max()


def test_residual_absorbs_bf16_branch_rounding():
    X, W, b = _tiny_problem()
    layer = O.prepare(W, b, O.calibration_absmax(X), 16)
    What = W * layer.lam[None, :]
    recon = layer.R + ((layer.lam[:, None] * layer.L1) @ layer.L2).T
    assert np.abs(recon - What).max() <= 2.0 ** -24 * np.abs(layer.R).max() * 1.0001


def test_golden_quantization_config():
    with open(os.path.join(HERE, "golden", "quantization_config.json")) as f:
        g = json.load(f)
    cfg = g["svdq_w4a4"]
    assert cfg["precision"] == "nvfp4"
    assert cfg["group_size"] == O.GROUP
    assert cfg["rank"] == CONFIGS["qkv"].rank


def test_tensor_scales_put_the_largest_group_scale_at_e4m3_max():
    # s_x from the calibration maxima equals the scale computed from the smoothed
    # activations themselves, and the largest group scale of X_hat and of R is 448.
    X, W, b = _tiny_problem()
    layer = O.prepare(W, b, O.calibration_absmax(X), 16)
    Xh = O.f32(X * layer.inv_lam[None, :])
    assert layer.s_x == float(O.f32(np.abs(Xh).max() / 2688.0))
    assert layer.s_w == float(O.f32(np.abs(layer.R).max() / 2688.0))
    _, xs, _ = O.quant_act_lora_down(X, layer)
    assert O.e4m3_decode(xs).max() == 448.0
    assert O.e4m3_decode(layer.w_scales).max() == 448.0


def test_smoothed_activations_are_single_fp32_products():
    # X_hat = fp32(X * inv_lambda): a bf16 input times an fp32 factor, rounded once to fp32
    # (numpy's float32 multiply is the independent statement); the chosen factors make products
    # that need more than bf16's 8 significant bits, so a 16-bit rounding of X_hat would show
    rng = np.random.default_rng(5)
    K = 64
    W = rng.normal(0, 0.02, (32, K)).astype(np.float32)
    layer = O.prepare(W, None, np.abs(rng.normal(size=K)) + 0.5, 0)
    inv = (1.0 + np.arange(1, K + 1) * 2.0 ** -12).astype(np.float32)
    layer.inv_lam = inv.astype(np.float64)
    Xb = f32_to_bf16_bits(rng.normal(size=(3, K)).astype(np.float32))
    X = bf16_bits_to_f32(Xb)
    want = (X * inv[None, :]).astype(np.float64)  # float32 x float32 -> float32
    got = O.smooth_activations(X.astype(np.float64), layer)
    np.testing.assert_array_equal(got, want)
    assert np.any(O.bf16_round(want) != want)
