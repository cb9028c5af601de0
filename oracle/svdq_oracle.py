"""fp64 CPU oracle for the SVDQuant NVFP4 W4A4 + low-rank linear.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this module.  The CUDA
library never calls it, and it shares no code with the CUDA library.

What it computes, in the order the method states it:

1. Outlier migration ("smoothing").  Svdq Int4 Flux.1 Canny Dev model card,
   "量化方法 -- SVDQuant / SVDQuant 概述", stage 2; "Nunchaku Lite in Diffusers"
   (Arabic translation), section "الخلفية: SVDQuant وNunchaku".  A per-input-channel
   factor lambda_j moves activation outliers into the weights:
   X_hat = X diag(lambda)^-1, W_hat = W diag(lambda).
   Reading: lambda_j = sqrt(max|X_j|) / sqrt(max|W_j|), calibrated on the run's X;
   lambda_j = 1 when either maximum is zero.
2. Low-rank split.  Same card, stage 3: W_hat^T = P S Q^T (SVD), the rank-r branch
   L1 = P_r S_r^1/2 (K x r), L2 = S_r^1/2 Q_r^T (r x N) runs in 16 bits (bf16), and the
   residual R = W_hat - (L1 L2)^T absorbs the rest, including the branch's bf16 rounding.
   Reading: the down-projection reads the layer input itself.  The engine notes of the
   same card, item (b), say that the down-projection and the quantizer consume the same
   input, so the smoothing is folded into the first factor once, offline:
   X_hat L1 = X (diag(lambda)^-1 L1).  The stored factor is L1s = bf16(diag(lambda)^-1 L1)
   and the residual is taken against the branch as stored,
   R = W_hat - (diag(lambda) L1s L2)^T.
3. 4-bit quantization of R and of X_hat.  "Nunchaku Lite in Diffusers", section
   "التحميل الأصلي في الناشرون" (the ``quantization_config`` block: precision nvfp4,
   group_size 16, rank 32).  NVFP4 = e2m1 codes, one e4m3 scale per 16 consecutive
   elements along K, and one fp32 tensor scale per tensor.
4. The layer output Y = Q(X_hat) Q(R)^T + (X L1s) L2 + b.

Beside the layer (each section below states its readings):
5. The fused QKV projection's output stage: per-head RMS normalization of Q and K and the rotary
   embedding ("Nunchaku Lite in Diffusers", section on structural rewrites) -- ``qk_norm_rope``.
6. The awq_w4a16 family: int4 weights in groups of 64 with fp16 scale and zero point times 16-bit
   activations, for the modulation projections (same page, kernel families and
   ``quantization_config``) -- ``awq_quantize``, ``awq_linear``.
7. The FLUX feed-forward pair: SVDQuant linear, GELU (tanh form), SVDQuant linear, with the
   intermediate kept unrounded when the pair is fused -- ``mlp_pair``.

Every fp32 operation of the method is emulated as "compute in fp64, round once to
fp32"; for + - * / and sqrt that equals the correctly rounded fp32 result (double
rounding from 53 to 24 bits is innocuous for these operations).  e4m3 (OCP E4M3FN:
max 448, subnormals down to 2^-9, no infinities) and e2m1 (magnitudes 0, 0.5, 1, 1.5,
2, 3, 4, 6) are rounded to nearest, ties to even, saturating to the largest finite
value.  A value that rounds to zero encodes as +0 in both formats.

Shapes: X (M, K), W (N, K) as in nn.Linear, b (N,), Y (M, N).
"""
from __future__ import annotations

import dataclasses

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0
GROUP = 16
# s = amax / (6 * 448) puts the largest group scale at the top of the e4m3 range.
TENSOR_SCALE_DIVISOR = E2M1_MAX * E4M3_MAX  # 2688

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


# --------------------------------------------------------------------------- rounding
def f32(x):
    """Round fp64 values to fp32 (nearest, ties to even); return them as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def _round_binary(x, p: int, emin: int):
    """Round to a binary format with p significant bits and smallest normal 2^emin.

    Subnormals share the quantum of the lowest binade.  np.rint rounds half to even.
    No overflow handling: callers saturate.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e = np.frexp(a)  # a = m 2^e with m in [0.5, 1)
    e = np.maximum(e - 1, emin)  # exponent of the binade holding a
    quantum = np.ldexp(1.0, e - (p - 1))
    q = np.rint(a / quantum) * quantum
    return np.copysign(q, x)


def bf16_round(x):
    """bf16 (8 significant bits) nearest-even rounding of fp64 values."""
    return _round_binary(x, 8, -126)


def e4m3_round(x):
    """OCP E4M3FN nearest-even rounding with saturation to +-448."""
    q = _round_binary(x, 4, -6)
    return np.clip(q, -E4M3_MAX, E4M3_MAX)


def e2m1_round(x):
    """e2m1 nearest-even rounding with saturation to +-6."""
    q = _round_binary(x, 2, 0)
    return np.clip(q, -E2M1_MAX, E2M1_MAX)


def e2m1_encode(v):
    """Encode e2m1 values (already on the grid) as 4-bit codes; zero is +0."""
    v = np.asarray(v, dtype=np.float64)
    mag = np.searchsorted(E2M1_MAGNITUDES, np.abs(v))
    if not np.all(E2M1_MAGNITUDES[np.minimum(mag, 7)] == np.abs(v)):
        raise ValueError("value not on the e2m1 grid")
    sign = (v < 0) & (mag > 0)
    return (mag | (sign.astype(np.int64) << 3)).astype(np.uint8)


def e2m1_decode(c):
    c = np.asarray(c, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[c & 7]
    return np.where(c & 8, -mag, mag)


def e4m3_encode(v):
    """Encode non-negative e4m3 values (on the grid) as 8-bit codes."""
    v = np.asarray(v, dtype=np.float64)
    if np.any(v < 0):
        raise ValueError("scales are non-negative")
    out = np.zeros(v.shape, dtype=np.uint8)
    nz = v > 0
    _, e = np.frexp(v[nz])
    e = e - 1
    normal = e >= -6
    ev = np.where(normal, e, -6)
    mant = np.where(normal, v[nz] / np.ldexp(1.0, ev) - 1.0, v[nz] / np.ldexp(1.0, -6))
    m3 = mant * 8.0
    if not np.all(m3 == np.round(m3)):
        raise ValueError("value not on the e4m3 grid")
    field = np.where(normal, ev + 7, 0)
    out[nz] = (field.astype(np.int64) << 3 | m3.astype(np.int64)).astype(np.uint8)
    return out


def e4m3_decode(c):
    c = np.asarray(c, dtype=np.int64)
    field = (c >> 3) & 0xF
    m = c & 7
    val = np.where(field == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.ldexp(1.0, field - 7))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return np.where(c & 0x80, -val, val)


# ----------------------------------------------------------------------- NVFP4
def tensor_scale(amax: float) -> float:
    """fp32 tensor scale s = amax / (6 * 448); s = 1 when amax is zero."""
    amax = float(amax)
    return 1.0 if amax == 0.0 else float(f32(amax / TENSOR_SCALE_DIVISOR))


def nvfp4_quantize(V, s: float):
    """Quantize the rows of V (fp32 values, K % 16 == 0) along K with tensor scale s.

    Per 16-element group: amax = max|v|; d = fp32(6 s); scale = e4m3(fp32(amax / d));
    if scale == 0 every code is +0; else eff = fp32(scale * s) and
    code_i = e2m1(fp32(v_i / eff)).
    Returns (codes uint8 [rows, K] holding 4-bit values, scale codes uint8 [rows, K/16]).
    """
    V = np.asarray(V, dtype=np.float64)
    rows, K = V.shape
    assert K % GROUP == 0
    G = V.reshape(rows, K // GROUP, GROUP)
    amax = np.abs(G).max(axis=2)
    d = f32(6.0 * s)
    sg = e4m3_round(f32(amax / d))
    eff = f32(sg * s)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = f32(G / eff[..., None])
    q = np.where(sg[..., None] == 0.0, 0.0, q)
    codes = e2m1_encode(e2m1_round(q)).reshape(rows, K)
    return codes, e4m3_encode(sg)


def nvfp4_dequantize(codes, scales):
    """Value of each element: e2m1(code) * e4m3(group scale) (tensor scale not applied)."""
    codes = np.asarray(codes)
    rows, K = codes.shape
    v = e2m1_decode(codes).reshape(rows, K // GROUP, GROUP)
    return (v * e4m3_decode(scales)[..., None]).reshape(rows, K)


def pack_codes(codes):
    """Two 4-bit codes per byte along K; element 2i in the low nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed):
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


# ----------------------------------------------------------------- smoothing
def smoothing_factors(a_x, a_w):
    """lambda_j = fp32(fp32(sqrt a_x) / fp32(sqrt a_w)); 1 where either max is zero.

    Returns (lambda, inv_lambda = fp32(1 / lambda)), fp32 values.
    """
    a_x = f32(a_x)
    a_w = f32(a_w)
    ok = (a_x > 0) & (a_w > 0)
    with np.errstate(divide="ignore", invalid="ignore"):
        lam = f32(f32(np.sqrt(a_x)) / f32(np.sqrt(a_w)))
    lam = np.where(ok, lam, 1.0)
    return lam, f32(1.0 / lam)


# ------------------------------------------------------------------- low rank
def svd_split(WhatT, rank: int):
    """Truncated SVD of W_hat^T (K x N): returns P_r (K x r), sigma_r, Q_r (N x r).

    Singular values descending.  Sign convention: the entry of largest magnitude in
    each column of P_r is positive (first such entry on ties); Q_r follows.
    """
    U, S, Vh = np.linalg.svd(np.asarray(WhatT, dtype=np.float64), full_matrices=False)
    P = U[:, :rank].copy()
    Q = Vh[:rank].T.copy()
    sig = S[:rank].copy()
    idx = np.argmax(np.abs(P), axis=0)
    sgn = np.sign(P[idx, np.arange(rank)])
    sgn[sgn == 0] = 1.0
    return P * sgn, sig, Q * sgn


@dataclasses.dataclass
class Layer:
    N: int
    K: int
    rank: int
    lam: np.ndarray  # (K,) fp32 values
    inv_lam: np.ndarray  # (K,)
    L1: np.ndarray  # (K, r) L1s = diag(lambda)^-1 P_r S_r^1/2: bf16 values (fp64 in "fp64" branch mode)
    L2: np.ndarray  # (r, N)
    R: np.ndarray  # (N, K) residual the weight quantizer sees (fp32 values)
    s_w: float
    s_x: float
    w_codes: np.ndarray  # (N, K) 4-bit codes
    w_scales: np.ndarray  # (N, K/16) e4m3 codes
    bias: np.ndarray  # (N,) fp32 values (zeros when absent)
    branch: str  # "bf16" (the method as run) or "fp64" (exact branch, invariant tests)


def prepare(W, b, a_x, rank: int, branch: str = "bf16", unit_lambda: bool = False) -> Layer:
    """Offline step: smoothing, SVD split, residual, weight quantization, scales.

    W (N, K) fp32 values, b (N,) or None, a_x (K,) calibration maxima max_m |X[m, j]|.
    ``branch="fp64"`` keeps L1, L2 and the residual unrounded (invariant tests only).
    ``unit_lambda`` forces lambda = 1 (plain W4A4 at rank 0).
    """
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    a_w = np.abs(W).max(axis=0)
    if unit_lambda:
        lam = np.ones(K)
        inv_lam = np.ones(K)
    else:
        lam, inv_lam = smoothing_factors(a_x, a_w)
    What = W * lam[None, :]  # exact in fp64: fp32 x fp32
    if rank > 0:
        P, sig, Q = svd_split(What.T, rank)
        rs = np.sqrt(sig)
        L1 = (P * rs[None, :]) / lam[:, None]  # smoothing folded into the first factor
        L2 = rs[:, None] * Q.T
        if branch == "bf16":
            L1 = bf16_round(L1)
            L2 = bf16_round(L2)
        R = What - ((lam[:, None] * L1) @ L2).T
    else:
        L1 = np.zeros((K, 0))
        L2 = np.zeros((0, N))
        R = What.copy()
    if branch == "bf16":
        R = f32(R)
    s_w = tensor_scale(f32(np.abs(R).max()))
    w_codes, w_scales = nvfp4_quantize(f32(R), s_w)
    ax_hat = f32(f32(a_x) * inv_lam)
    s_x = tensor_scale(ax_hat.max())
    bias = np.zeros(N) if b is None else f32(b)
    return Layer(N, K, rank, lam, inv_lam, L1, L2, R, s_w, s_x, w_codes, w_scales, bias, branch)


# ------------------------------------------------------------------ forward
def smooth_activations(Xv, layer: Layer):
    """X_hat = fp32(X * inv_lambda) per element (fp64 X / lambda in "fp64" branch mode)."""
    Xv = np.asarray(Xv, dtype=np.float64)
    if layer.branch == "fp64":
        return Xv / layer.lam[None, :]
    return f32(Xv * layer.inv_lam[None, :])


def quant_act_lora_down(Xv, layer: Layer):
    """Activation side of the layer: NVFP4 codes/scales of X_hat and La = X L1s.

    The down-projection reads the layer input X (bf16 values, exact in fp64) against the
    smoothing-folded factor L1s, so La = X_hat L1 up to the rounding of L1s; La is kept
    in fp64.  Returns (codes [M, K], scale codes [M, K/16], La [M, r]).
    """
    Xv = np.asarray(Xv, dtype=np.float64)
    Xh = smooth_activations(Xv, layer)
    codes, scales = nvfp4_quantize(f32(Xh), layer.s_x)
    if layer.rank:
        La = Xv @ layer.L1
    else:
        La = np.zeros((Xh.shape[0], 0))
    return codes, scales, La


def gemm_w4a4_lora_up(x_codes, x_scales, La, layer: Layer):
    """Y = s_x s_w deq(Q(X_hat)) deq(Q(R))^T + La L2 + b, all in fp64."""
    Xd = nvfp4_dequantize(x_codes, x_scales)
    Wd = nvfp4_dequantize(layer.w_codes, layer.w_scales)
    Y = (layer.s_x * layer.s_w) * (Xd @ Wd.T)
    if layer.rank:
        Y = Y + La @ layer.L2
    return Y + layer.bias[None, :]


def layer_forward(Xv, layer: Layer):
    xc, xs, La = quant_act_lora_down(Xv, layer)
    return gemm_w4a4_lora_up(xc, xs, La, layer)


def calibration_absmax(Xv):
    """a_x[j] = max_m |X[m, j]| (exact)."""
    return np.abs(np.asarray(Xv, dtype=np.float64)).max(axis=0)


# --------------------------------------------------------------------------- fused QKV output stage
# "Nunchaku Lite in Diffusers", section on quantized models with structural rewrites
# ("نماذج الكم مع إعادة الكتابة الهيكلية"): FLUX.1-dev's Q, K and V projections are
# concatenated along the output dimension, in that order, into one to_qkv layer, and the
# engine's fused operator consumes that projection together with the Q/K normalization
# (norm_q, norm_k) and the rotary embedding (apply_rotary_emb on Q and K), which the default
# path runs as separate steps after splitting the output into heads.
# Readings (the page names the steps, not their formulas):
#   * Y = [Q | K | V], each section `heads` heads of `head_dim` columns, head h of a section
#     in columns h*head_dim .. (h+1)*head_dim - 1;
#   * norm_q / norm_k are RMS normalizations over a head's head_dim values with a learned
#     per-column weight: u = y w / sqrt(mean(y^2) + eps);
#   * the rotary embedding turns each pair of columns (2i, 2i + 1) of a Q or K head by the
#     angle theta[m, i] of token m and pair i, given as the table (cos theta, sin theta);
#   * V passes through unchanged;
#   * in the fused operator the normalization reads the layer output before its 16-bit
#     rounding.
def rms_norm_heads(Yh, weight, eps: float):
    """u = y * w / sqrt(mean(y^2) + eps) over the last axis (one head), fp64."""
    Yh = np.asarray(Yh, dtype=np.float64)
    ms = np.mean(Yh * Yh, axis=-1, keepdims=True)
    return Yh / np.sqrt(ms + eps) * np.asarray(weight, dtype=np.float64)


def rotary_pairs(U, cos, sin):
    """Turn the pairs (U[..., 2i], U[..., 2i+1]) by the angle whose cosine and sine are
    cos[m, i], sin[m, i]; U is (M, heads, head_dim), cos / sin are (M, head_dim / 2)."""
    U = np.asarray(U, dtype=np.float64)
    x0 = U[..., 0::2]
    x1 = U[..., 1::2]
    c = np.asarray(cos, dtype=np.float64)[:, None, :]
    s = np.asarray(sin, dtype=np.float64)[:, None, :]
    out = np.empty_like(U)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x1 * c + x0 * s
    return out


def qk_norm_rope(Y, heads: int, head_dim: int, norm_q_weight, norm_k_weight, cos, sin, eps: float):
    """Output stage of the fused QKV projection: per-head RMS normalization and rotary
    embedding of the Q and K sections of Y = [Q | K | V]; V unchanged. fp64."""
    Y = np.asarray(Y, dtype=np.float64)
    M, N = Y.shape
    width = heads * head_dim
    assert N == 3 * width and head_dim % 2 == 0
    Z = Y.copy()
    for sec, w in ((0, norm_q_weight), (1, norm_k_weight)):
        block = Y[:, sec * width:(sec + 1) * width].reshape(M, heads, head_dim)
        U = rms_norm_heads(block, w, eps)
        Z[:, sec * width:(sec + 1) * width] = rotary_pairs(U, cos, sin).reshape(M, width)
    return Z


# --------------------------------------------------------------------------- awq_w4a16
# "Nunchaku Lite in Diffusers": the second kernel family, awq_w4a16 (4-bit weights, 16-bit
# activations), serves the adaptive-normalization / modulation projections (FLUX's
# adaLN_modulation), which are memory-bound and precision-sensitive; its quantization_config
# entry fixes precision int4 and group_size 64.
# Readings (the page gives no formulas):
#   * groups of 64 consecutive input channels of a weight row share one scale and one zero
#     point (AWQ's asymmetric storage): W_hat[n, k] = (q[n, k] - z[n, g]) * s[n, g], q and z in
#     0 .. 15, s stored as fp16;
#   * the codes come from round-to-nearest on the group's range, decided in fp32:
#       range = fp32(max - min), raised to fp32(1e-5) when smaller;
#       s = fp16(fp32(range / 15));
#       z = clamp(rint(fp32(-min / s)), 0, 15);   q = clamp(rint(fp32(w / s)) + z, 0, 15)
#     (rint: nearest, ties to even).  AWQ's activation-aware search for per-channel scales is a
#     calibration procedure the pages do not describe; it would change W before this step.
#   * Y = X W_hat^T + b with 16-bit X and the output rounded to bf16 once.
AWQ_GROUP = 64


def f16(x):
    """Round fp64 values to fp16 (nearest, ties to even); return them as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def awq_quantize(W, group: int = AWQ_GROUP):
    """Int4 codes q (N, K) uint8, fp16 scales s (N, K/group) as fp64, zeros z (N, K/group) uint8."""
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    G = W.reshape(N, K // group, group)
    mx = G.max(axis=2)
    mn = G.min(axis=2)
    rng = f32(mx - mn)
    rng = np.where(rng < f32(1e-5), f32(1e-5), rng)
    s = f16(f32(rng / 15.0))
    z = np.clip(np.rint(f32(-mn / s)), 0, 15)
    q = np.clip(np.rint(f32(G / s[:, :, None])) + z[:, :, None], 0, 15)
    return q.reshape(N, K).astype(np.uint8), s, z.astype(np.uint8)


def awq_dequantize(q, s, z, group: int = AWQ_GROUP):
    N, K = q.shape
    qg = q.reshape(N, K // group, group).astype(np.float64)
    return ((qg - z[:, :, None].astype(np.float64)) * s[:, :, None]).reshape(N, K)


def awq_linear(Xv, q, s, z, bias=None, group: int = AWQ_GROUP):
    """Y = X W_hat^T + b in fp64 (W_hat the dequantized int4 weight)."""
    Y = np.asarray(Xv, dtype=np.float64) @ awq_dequantize(q, s, z, group).T
    return Y if bias is None else Y + np.asarray(bias, dtype=np.float64)[None, :]


# --------------------------------------------------------------------------- MLP pair
# "Nunchaku Lite in Diffusers" lists fused GELU / MLP kernels among the engine's fusions; FLUX's
# feed-forward is Linear(3072 -> 12288), GELU (tanh form), Linear(12288 -> 3072), both linears
# SVDQuant layers. Reading: in the fused pair the intermediate H = GELU(Y1) reaches the second
# layer's quantizer and low-rank branch without a 16-bit rounding (it stays on chip); in the
# unfused pair H is written to memory between the layers, as bf16. The second layer is calibrated
# on H (its smoothing factors come from max |H_j|). The down layer's activation codes are decided
# by floating point (the GELU), so a fused kernel's parity is judged at the pair's output.
def gelu_tanh(x):
    """0.5 x (1 + tanh(sqrt(2 / pi) (x + 0.044715 x^3))), fp64."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def mlp_hidden(Xv, up: Layer, fused: bool = True):
    """H = GELU(first layer's output), rounded to bf16 when the pair is not fused."""
    codes, scales, La = quant_act_lora_down(Xv, up)
    H = gelu_tanh(gemm_w4a4_lora_up(codes, scales, La, up))
    return H if fused else bf16_round(H)


def mlp_pair(Xv, up: Layer, down: Layer, fused: bool = True):
    """Z = down(GELU(up(X))) with both linears the SVDQuant layer, fp64."""
    H = mlp_hidden(Xv, up, fused)
    codes, scales, La = quant_act_lora_down(H, down)
    return gemm_w4a4_lora_up(codes, scales, La, down)
