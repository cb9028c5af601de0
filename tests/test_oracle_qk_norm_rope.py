"""Pins of the oracle's fused-QKV output stage (per-head Q/K RMS normalization and rotary
embedding) to a library routine, an independent complex-number statement, closed forms
and invariants ("Nunchaku Lite in Diffusers", section on structural rewrites: the fused
to_qkv projection whose operator also applies norm_q, norm_k and the rotary embedding)."""
import numpy as np
import pytest
import torch

from oracle import svdq_oracle as O
from synth import qk_norm_weights, rope_table

H, D = 2, 128


def _y(M=5, seed=0, scale=3.0):
    return np.random.default_rng(seed).normal(0.0, scale, (M, 3 * H * D))


def test_rms_norm_matches_torch_rms_norm():
    Y = _y(7).reshape(7, 3 * H, D)
    w = qk_norm_weights(D)[0].astype(np.float64)
    want = torch.nn.functional.rms_norm(torch.from_numpy(Y), (D,), torch.from_numpy(w), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rms_norm_heads(Y, w, 1e-6), want, rtol=1e-13, atol=1e-13)


def test_rotary_is_complex_multiplication():
    rng = np.random.default_rng(1)
    U = rng.normal(size=(6, H, D))
    ang = rng.uniform(-np.pi, np.pi, (6, D // 2))
    z = (U[..., 0::2] + 1j * U[..., 1::2]) * np.exp(1j * ang)[:, None, :]
    got = O.rotary_pairs(U, np.cos(ang), np.sin(ang))
    np.testing.assert_allclose(got[..., 0::2], z.real, rtol=0, atol=1e-13)
    np.testing.assert_allclose(got[..., 1::2], z.imag, rtol=0, atol=1e-13)


def test_rotary_quarter_turn_and_identity():
    U = np.random.default_rng(2).normal(size=(3, H, D))
    one, zero = np.ones((3, D // 2)), np.zeros((3, D // 2))
    np.testing.assert_array_equal(O.rotary_pairs(U, one, zero), U)
    q = O.rotary_pairs(U, zero, one)
    np.testing.assert_array_equal(q[..., 0::2], -U[..., 1::2])
    np.testing.assert_array_equal(q[..., 1::2], U[..., 0::2])


def test_rotary_depends_on_relative_position_only():
    # angle = position x frequency: <R(p) q, R(p') k> is unchanged when both positions shift
    rng = np.random.default_rng(3)
    q, k = rng.normal(size=(1, 1, D)), rng.normal(size=(1, 1, D))
    freq = 10000.0 ** (-np.arange(0, D, 2) / D)

    def rot(x, pos):
        a = (pos * freq)[None, :]
        return O.rotary_pairs(x, np.cos(a), np.sin(a))

    d0 = np.sum(rot(q, 5.0) * rot(k, 2.0))
    d1 = np.sum(rot(q, 45.0) * rot(k, 42.0))
    assert abs(d0 - d1) < 1e-10 * np.sum(np.abs(q) * np.abs(k))
    assert abs(np.sum(rot(q, 5.0) * rot(k, 3.0)) - d0) > 1e-3  # and it does depend on it


def test_sections_closed_form():
    # zero angles, eps = 0, constant weights 2 (Q) and 3 (K): every Q head has rms exactly 2,
    # every K head rms 3, and V passes through bit for bit
    Y = _y(4)
    M = Y.shape[0]
    one, zero = np.ones((M, D // 2)), np.zeros((M, D // 2))
    Z = O.qk_norm_rope(Y, H, D, np.full(D, 2.0), np.full(D, 3.0), one, zero, 0.0)
    rms = np.sqrt(np.mean(Z[:, :2 * H * D].reshape(M, 2, H, D) ** 2, axis=-1))
    np.testing.assert_allclose(rms[:, 0], 2.0, rtol=1e-14)
    np.testing.assert_allclose(rms[:, 1], 3.0, rtol=1e-14)
    np.testing.assert_array_equal(Z[:, 2 * H * D:], Y[:, 2 * H * D:])


def test_scale_invariance_and_eps():
    Y = _y(4)
    wq, wk = (w.astype(np.float64) for w in qk_norm_weights(D))
    t = rope_table(4, D, n_text=1).astype(np.float64)
    c, s = t[..., 0], t[..., 1]
    Z1 = O.qk_norm_rope(Y, H, D, wq, wk, c, s, 0.0)
    Z2 = O.qk_norm_rope(7.5 * Y, H, D, wq, wk, c, s, 0.0)
    np.testing.assert_allclose(Z2[:, :2 * H * D], Z1[:, :2 * H * D], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(Z2[:, 2 * H * D:], 7.5 * Y[:, 2 * H * D:], rtol=1e-15)
    # eps only matters against a small mean square: a head of zeros stays zero
    Y0 = Y.copy()
    Y0[:, :D] = 0.0
    Z0 = O.qk_norm_rope(Y0, H, D, wq, wk, c, s, 1e-6)
    assert np.all(Z0[:, :D] == 0.0)


def test_pair_norms_survive_rotation():
    Y = _y(6)
    wq, wk = (w.astype(np.float64) for w in qk_norm_weights(D))
    t = rope_table(6, D, n_text=2).astype(np.float64)
    Zr = O.qk_norm_rope(Y, H, D, wq, wk, t[..., 0], t[..., 1], 1e-6)
    Zn = O.qk_norm_rope(Y, H, D, wq, wk, np.ones((6, D // 2)), np.zeros((6, D // 2)), 1e-6)
    n_r = Zr[:, :2 * H * D][:, 0::2] ** 2 + Zr[:, :2 * H * D][:, 1::2] ** 2
    n_n = Zn[:, :2 * H * D][:, 0::2] ** 2 + Zn[:, :2 * H * D][:, 1::2] ** 2
    # the fp32 table has cos^2 + sin^2 = 1 only to within 2^-23
    np.testing.assert_allclose(n_r, n_n, rtol=3e-7, atol=1e-14)


def test_rope_table_recipe():
    t = rope_table(4608)
    assert t.shape == (4608, 64, 2) and t.dtype == np.float32
    # text tokens sit at position 0; cos^2 + sin^2 = 1 to fp32 precision
    assert np.all(t[:512, :, 0] == 1.0) and np.all(t[:512, :, 1] == 0.0)
    np.testing.assert_allclose(t[..., 0].astype(np.float64) ** 2 + t[..., 1].astype(np.float64) ** 2, 1.0, atol=2e-7)
    # image token (row 1, column 3): pair 8 is the row axis at frequency 1, pair 36 the column axis
    m = 512 + 64 + 3
    assert t[m, 8, 1] == np.float32(np.sin(1.0)) and t[m, 36, 1] == np.float32(np.sin(3.0))
    assert t[m, 0, 0] == 1.0


@pytest.mark.parametrize("plant", ["swap_weights", "rotate_minus", "mean_not_rms", "skip_v"])
def test_pins_catch_planted_mistakes(plant, monkeypatch):
    """Each planted mistake in a copy of the oracle's stage must change its output on the
    pinned cases above."""
    Y = _y(4)
    wq, wk = (w.astype(np.float64) for w in qk_norm_weights(D))
    t = rope_table(4, D, n_text=1).astype(np.float64)
    c, s = t[..., 0], t[..., 1]
    good = O.qk_norm_rope(Y, H, D, wq, wk, c, s, 1e-6)
    if plant == "swap_weights":
        bad = O.qk_norm_rope(Y, H, D, wk, wq, c, s, 1e-6)
    elif plant == "rotate_minus":
        bad = O.qk_norm_rope(Y, H, D, wq, wk, c, -s, 1e-6)
    elif plant == "mean_not_rms":
        monkeypatch.setattr(O, "rms_norm_heads", lambda Yh, w, eps: Yh / np.sqrt(np.abs(np.mean(Yh, -1, keepdims=True)) + eps) * w)
        bad = O.qk_norm_rope(Y, H, D, wq, wk, c, s, 1e-6)
    else:
        bad = good.copy()
        bad[:, 2 * H * D:] = 0.0
    assert not np.allclose(bad, good)
