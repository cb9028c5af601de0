"""Pins of the oracle's MLP-pair statement (FLUX feed-forward: SVDQuant linear, GELU in its tanh
form, SVDQuant linear; the fused pair keeps the intermediate unrounded) to torch's GELU, an exact
identity of the tanh form, and the textbook MLP that the pair reduces to at full rank."""
import numpy as np
import torch

from oracle import svdq_oracle as O


def test_gelu_matches_torch_tanh_form():
    x = np.linspace(-8.0, 8.0, 2001)
    want = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    np.testing.assert_allclose(O.gelu_tanh(x), want, rtol=1e-14, atol=1e-15)


def test_gelu_odd_part_is_x():
    # 0.5 x (1 + t(x)) - 0.5 (-x) (1 + t(-x)) = x because tanh is odd
    x = np.random.default_rng(0).normal(0, 3, 1000)
    np.testing.assert_allclose(O.gelu_tanh(x) - O.gelu_tanh(-x), x, rtol=1e-14, atol=1e-15)
    assert O.gelu_tanh(np.array([0.0]))[0] == 0.0
    assert abs(O.gelu_tanh(np.array([12.0]))[0] - 12.0) < 1e-12


def _pair(M=48, D=64, F=256, seed=0, branch="fp64", full=True):
    rng = np.random.default_rng(seed)
    X = rng.normal(size=(M, D))
    W1 = rng.normal(0, 0.1, (F, D)).astype(np.float32)
    b1 = rng.normal(0, 0.01, F).astype(np.float32)
    W2 = rng.normal(0, 0.05, (D, F)).astype(np.float32)
    b2 = rng.normal(0, 0.01, D).astype(np.float32)
    up = O.prepare(W1, b1, O.calibration_absmax(X), min(D, F) if full else 16, branch=branch)
    H = O.mlp_hidden(X, up)
    down = O.prepare(W2, b2, O.calibration_absmax(H), min(D, F) if full else 16, branch=branch)
    return X, W1, b1, W2, b2, up, down


def test_full_rank_pair_is_the_textbook_mlp():
    # at full rank with an exact (fp64) branch the residuals vanish, so each layer is X W^T + b
    # and the pair is W2 GELU(W1 x + b1) + b2
    X, W1, b1, W2, b2, up, down = _pair()
    want = O.gelu_tanh(X @ W1.T.astype(np.float64) + b1) @ W2.T.astype(np.float64) + b2
    got = O.mlp_pair(X, up, down)
    assert np.max(np.abs(got - want)) <= 1e-9 * np.max(np.abs(want))


def test_unfused_pair_rounds_the_intermediate():
    X, W1, b1, W2, b2, up, down = _pair(branch="bf16", full=False)
    Hf = O.mlp_hidden(X, up, fused=True)
    Hu = O.mlp_hidden(X, up, fused=False)
    # bf16 keeps 8 significant bits (unit roundoff 2^-8): the rounding moves H by at most 2^-8
    # relative, and does move it
    assert np.all(np.abs(Hu - Hf) <= 2.0 ** -8 * np.abs(Hf) * (1 + 1e-12))
    assert np.any(Hu != Hf)
    Zf, Zu = O.mlp_pair(X, up, down, fused=True), O.mlp_pair(X, up, down, fused=False)
    rel = np.linalg.norm(Zu - Zf) / np.linalg.norm(Zf)
    assert 0.0 < rel < 0.05
