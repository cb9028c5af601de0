"""Seeded synthetic inputs for the SVDQuant NVFP4 W4A4 + low-rank linear.

This module only draws random numbers and rounds the activations to bf16 storage.
It holds none of the method's arithmetic (no smoothing, SVD, quantization or GEMM),
so both the fp64 oracle and the CUDA library can consume its outputs.

Shapes follow the FLUX-like linear layers of the workloads: a tiny layer, the fused
QKV projection (N = 3 x 3072, the ``to_qkv`` module that concatenates Q, K and V along
the output dimension, "Nunchaku Lite in Diffusers" page, section on structural rewrites),
the MLP up/down pair, a token-count sweep and a rank sweep.

Recipe (every config uses ``numpy.random.Generator(PCG64(seed))``, seed 0 unless given).
Draw order: outlier channel indices, outlier factors, activations, weights, bias.

* ``tiny`` / ``sweep_m`` / ``sweep_r``: X ~ N(0, 1); 4 input channels drawn without
  replacement are scaled by 30. W ~ N(0, 0.02^2); the same 4 columns scaled by 0.2.
  b ~ N(0, 0.01^2).
* ``qkv``: X ~ N(0, 1); 1% of the channels (31 of 3072) scaled by a factor U[20, 50]
  each. W as above (outlier columns x 0.2). b ~ N(0, 0.01^2).
* ``mlp_up``: Z ~ N(0, 1) per row layer-normed (no affine, eps 1e-6), then 1% of the
  channels scaled by U[20, 50]. W, b as ``qkv``.
* ``mlp_down``: GELU (erf form) of Z ~ N(0, 1) on 99.5% of the channels; the other 0.5%
  (61 of 12288) are LogNormal(0, 1.5^2) draws (non-negative, heavy tailed). W, b as ``qkv``.

Activations are generated in fp64, cast to fp32 and rounded to bf16 (round to nearest
even) for storage; W and b are stored as fp32.

Inputs of the fused QKV output stage (per-head Q/K normalization and rotary embedding):
``rope_table`` gives FLUX-like token positions (text tokens first at position 0, then image
tokens on a 64-wide latent grid, three position axes of 16, 56 and 56 head columns, base
10000) as a (cos, sin) table per token and column pair, angles in fp64 rounded to fp32;
``qk_norm_weights`` draws the two normalization weight vectors ~ N(1, 0.1^2).

Inputs of the 4-bit-weight modulation projection (awq_w4a16): FLUX's adaptive-normalization
linear reads SiLU of the conditioning embedding, so X = SiLU(Z), Z ~ N(0, 1), rounded to bf16;
W ~ N(0, 0.02^2) fp32, b ~ N(0, 0.01^2) (``make_modulation_inputs``).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "LayerShape",
    "CONFIGS",
    "config_shape",
    "make_inputs",
    "f32_to_bf16_bits",
    "bf16_bits_to_f32",
    "rope_table",
    "qk_norm_weights",
    "make_modulation_inputs",
]


@dataclasses.dataclass(frozen=True)
class LayerShape:
    name: str
    M: int
    K: int
    N: int
    rank: int
    x_kind: str  # "spiky4", "spiky1pct", "layernorm1pct", "gelu_lognormal"


# Named workloads (FLUX-like linear shapes).
CONFIGS = {
    "tiny": LayerShape("tiny", 256, 512, 512, 16, "spiky4"),
    "qkv": LayerShape("qkv", 4608, 3072, 9216, 32, "spiky1pct"),
    "mlp_up": LayerShape("mlp_up", 4608, 3072, 12288, 32, "layernorm1pct"),
    "mlp_down": LayerShape("mlp_down", 4608, 12288, 3072, 32, "gelu_lognormal"),
}
for _m in (256, 1024, 4096, 16384):
    CONFIGS[f"sweep_m{_m}"] = LayerShape(f"sweep_m{_m}", _m, 3072, 3072, 32, "spiky4")
for _r in (0, 16, 32, 64, 128):
    CONFIGS[f"sweep_r{_r}"] = LayerShape(f"sweep_r{_r}", 4608, 3072, 3072, _r, "spiky4")


def config_shape(name: str) -> LayerShape:
    return CONFIGS[name]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _gelu_erf(z: np.ndarray) -> np.ndarray:
    from scipy.special import erf

    return 0.5 * z * (1.0 + erf(z / math.sqrt(2.0)))


def make_inputs(shape: LayerShape, seed: int = 0, M: int | None = None):
    """Return (X_bf16_bits[M,K] uint16, W[N,K] float32, b[N] float32, outlier_channels).

    ``M`` overrides the token count (the weights do not depend on it, the activations
    are drawn with the same recipe).
    """
    M = shape.M if M is None else int(M)
    K, N = shape.K, shape.N
    rng = np.random.Generator(np.random.PCG64(seed))

    if shape.x_kind == "spiky4":
        ch = rng.choice(K, 4, replace=False)
        fac = np.full(4, 30.0)
    elif shape.x_kind in ("spiky1pct", "layernorm1pct"):
        n_out = int(round(0.01 * K))
        ch = rng.choice(K, n_out, replace=False)
        fac = rng.uniform(20.0, 50.0, n_out)
    elif shape.x_kind == "gelu_lognormal":
        n_out = int(round(0.005 * K))
        ch = rng.choice(K, n_out, replace=False)
        fac = None
    else:  # pragma: no cover - table above is closed
        raise ValueError(shape.x_kind)

    if shape.x_kind == "spiky4" or shape.x_kind == "spiky1pct":
        X = rng.standard_normal((M, K))
        X[:, ch] *= fac
    elif shape.x_kind == "layernorm1pct":
        Z = rng.standard_normal((M, K))
        mu = Z.mean(axis=1, keepdims=True)
        var = Z.var(axis=1, keepdims=True)
        X = (Z - mu) / np.sqrt(var + 1e-6)
        X[:, ch] *= fac
    else:
        Z = rng.standard_normal((M, K))
        X = _gelu_erf(Z)
        X[:, ch] = rng.lognormal(0.0, 1.5, (M, len(ch)))

    W = rng.normal(0.0, 0.02, (N, K))
    W[:, ch] *= 0.2
    b = rng.normal(0.0, 0.01, N)

    Xb = f32_to_bf16_bits(X.astype(np.float32))
    return Xb, W.astype(np.float32), b.astype(np.float32), np.sort(ch)


def rope_table(M: int, head_dim: int = 128, n_text: int | None = None, grid_w: int = 64,
               axes=(16, 56, 56), theta: float = 10000.0) -> np.ndarray:
    """(cos, sin) of the rotary angle per token and head-column pair: float32 [M, head_dim/2, 2].

    Token m < n_text is a text token (every position coordinate 0); token n_text + j is the
    image token at row j // grid_w, column j % grid_w of the latent grid, with coordinates
    (0, row, column) on the three axes. Axis a of width d_a contributes d_a / 2 pairs with
    frequencies theta^(-2k / d_a), k = 0 .. d_a/2 - 1; the angle is coordinate x frequency.
    ``n_text`` defaults to the FLUX proportion of 512 text tokens per 4608.
    """
    assert sum(axes) == head_dim and all(d % 2 == 0 for d in axes)
    if n_text is None:
        n_text = (M * 512) // 4608
    m = np.arange(M)
    j = np.maximum(m - n_text, 0)
    img = m >= n_text
    coords = np.stack([np.zeros(M), np.where(img, j // grid_w, 0), np.where(img, j % grid_w, 0)], axis=1)
    angles = []
    for a, d in enumerate(axes):
        freq = theta ** (-np.arange(0, d, 2, dtype=np.float64) / d)
        angles.append(coords[:, a:a + 1].astype(np.float64) * freq[None, :])
    ang = np.concatenate(angles, axis=1)
    return np.stack([np.cos(ang), np.sin(ang)], axis=-1).astype(np.float32)


def qk_norm_weights(head_dim: int = 128, seed: int = 0):
    """Weights of the Q and K normalizations, float32 [head_dim] each, ~ N(1, 0.1^2)."""
    rng = np.random.Generator(np.random.PCG64(seed + 1000))
    return (rng.normal(1.0, 0.1, head_dim).astype(np.float32), rng.normal(1.0, 0.1, head_dim).astype(np.float32))


def make_modulation_inputs(M: int, K: int, N: int, seed: int = 0):
    """(X_bf16_bits [M, K] uint16, W [N, K] float32, b [N] float32) for a modulation projection."""
    rng = np.random.Generator(np.random.PCG64(seed + 2000))
    Z = rng.standard_normal((M, K))
    X = Z / (1.0 + np.exp(-Z))
    W = rng.normal(0.0, 0.02, (N, K))
    b = rng.normal(0.0, 0.01, N)
    return f32_to_bf16_bits(X.astype(np.float32)), W.astype(np.float32), b.astype(np.float32)
