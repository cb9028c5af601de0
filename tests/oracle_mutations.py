"""Planted mistakes for the oracle, applied to the module on the CPU (never to the CUDA path)
when the environment names one (SVDQ_ORACLE_MUTATION); tests/test_oracle_mutations.py checks
that the pins in tests/test_oracle_pins.py catch every one of them."""
import numpy as np


def _apply(O, name):
    orig_round = O._round_binary
    orig_smooth = O.smoothing_factors
    orig_svd = O.svd_split
    orig_prepare = O.prepare
    orig_gemm = O.gemm_w4a4_lora_up

    if name == "ties_away_from_zero":
        def rb(x, p, emin):
            x = np.asarray(x, dtype=np.float64)
            a = np.abs(x)
            _, e = np.frexp(a)
            e = np.maximum(e - 1, emin)
            quantum = np.ldexp(1.0, e - (p - 1))
            return np.copysign(np.floor(a / quantum + 0.5) * quantum, x)
        O._round_binary = rb
    elif name == "bias_dropped":
        O.gemm_w4a4_lora_up = lambda xc, xs, La, layer: orig_gemm(xc, xs, La, layer) - layer.bias[None, :]
    elif name == "branch_sign":
        def svd(WhatT, rank):
            P, sig, Q = orig_svd(WhatT, rank)
            return P, sig, -Q  # L2 negated: the residual adds the branch instead of removing it
        O.svd_split = svd
    elif name == "tensor_scale_divisor":
        O.TENSOR_SCALE_DIVISOR = 448.0
    elif name == "lambda_inverted":
        def sm(a_x, a_w):
            lam, inv = orig_smooth(a_x, a_w)
            return inv, lam
        O.smoothing_factors = sm
    elif name == "no_sign_convention":
        def svd(WhatT, rank):
            U, S, Vh = np.linalg.svd(np.asarray(WhatT, dtype=np.float64), full_matrices=False)
            P, Q = -U[:, :rank], -Vh[:rank].T
            return P, S[:rank], Q
        O.svd_split = svd
    elif name == "e4m3_two_mantissa_bits":
        O.e4m3_round = lambda x: np.clip(orig_round(x, 3, -6), -O.E4M3_MAX, O.E4M3_MAX)
    elif name == "e4m3_max_240":
        O.E4M3_MAX = 240.0
    elif name == "bf16_smoothed_activations":
        O.smooth_activations = lambda Xv, layer: O.bf16_round(np.asarray(Xv, dtype=np.float64) * layer.inv_lam[None, :])
    elif name == "alpha_without_s_w":
        def gemm(xc, xs, La, layer):
            Xd = O.nvfp4_dequantize(xc, xs)
            Wd = O.nvfp4_dequantize(layer.w_codes, layer.w_scales)
            Y = layer.s_x * (Xd @ Wd.T)
            if layer.rank:
                Y = Y + La @ layer.L2
            return Y + layer.bias[None, :]
        O.gemm_w4a4_lora_up = gemm
    elif name == "s_x_unsmoothed":
        def prep(W, b, a_x, rank, branch="bf16", unit_lambda=False):
            L = orig_prepare(W, b, a_x, rank, branch, unit_lambda)
            L.s_x = O.tensor_scale(O.f32(a_x).max())
            return L
        O.prepare = prep
    elif name == "nibble_order":
        O.pack_codes = lambda c: (np.asarray(c, np.uint8)[:, 1::2] | (np.asarray(c, np.uint8)[:, 0::2] << 4)).astype(np.uint8)
    elif name == "no_zero_guard":
        def sm(a_x, a_w):
            a_x, a_w = O.f32(a_x), O.f32(a_w)
            with np.errstate(divide="ignore", invalid="ignore"):
                lam = O.f32(O.f32(np.sqrt(a_x)) / O.f32(np.sqrt(a_w)))
                return lam, O.f32(1.0 / lam)
        O.smoothing_factors = sm
    elif name == "unbalanced_split":
        def svd(WhatT, rank):
            P, sig, Q = orig_svd(WhatT, rank)
            r = np.sqrt(sig)
            return P * r[None, :], sig, Q / r[None, :]  # L1 = P S, L2 = Q^T
        O.svd_split = svd
    # fused QKV output stage
    elif name == "rope_turns_backwards":
        orig = O.rotary_pairs
        O.rotary_pairs = lambda U, cos, sin: orig(U, cos, -np.asarray(sin))
    elif name == "rms_without_eps_inside_sqrt":
        O.rms_norm_heads = lambda Yh, w, eps: np.asarray(Yh, np.float64) / (
            np.sqrt(np.mean(np.asarray(Yh, np.float64) ** 2, axis=-1, keepdims=True)) + eps) * np.asarray(w, np.float64)
    elif name == "rope_pairs_split_halves":
        def rot(U, cos, sin):  # pairs (i, i + D/2) instead of (2i, 2i + 1)
            U = np.asarray(U, np.float64)
            h = U.shape[-1] // 2
            x0, x1 = U[..., :h], U[..., h:]
            c, sn = np.asarray(cos)[:, None, :], np.asarray(sin)[:, None, :]
            return np.concatenate([x0 * c - x1 * sn, x1 * c + x0 * sn], axis=-1)
        O.rotary_pairs = rot
    # awq_w4a16
    elif name == "awq_zero_point_added":
        O.awq_dequantize = lambda q, s, z, group=64: ((q.reshape(q.shape[0], -1, group).astype(np.float64)
                                                        + z[:, :, None]) * s[:, :, None]).reshape(q.shape)
    elif name == "awq_scale_not_fp16":
        O.f16 = lambda x: np.asarray(x, dtype=np.float64)
    elif name == "awq_ties_away":
        orig_q = O.awq_quantize

        def aq(W, group=64):
            saved = np.rint
            np.rint = lambda x: np.floor(np.asarray(x) + 0.5)
            try:
                return orig_q(W, group)
            finally:
                np.rint = saved
        O.awq_quantize = aq
    # MLP pair
    elif name == "gelu_erf_form":
        from math import erf
        O.gelu_tanh = lambda x: 0.5 * np.asarray(x, np.float64) * (1.0 + np.vectorize(erf)(np.asarray(x, np.float64) / np.sqrt(2.0)))
    elif name == "mlp_unfused_not_rounded":
        orig_h = O.mlp_hidden
        O.mlp_hidden = lambda Xv, up, fused=True: orig_h(Xv, up, True)
    else:
        raise ValueError(name)


# mistake -> the pin file that must catch it
PIN_FILES = {
    "rope_turns_backwards": "tests/test_oracle_qk_norm_rope.py",
    "rms_without_eps_inside_sqrt": "tests/test_oracle_qk_norm_rope.py",
    "rope_pairs_split_halves": "tests/test_oracle_qk_norm_rope.py",
    "awq_zero_point_added": "tests/test_oracle_awq.py",
    "awq_scale_not_fp16": "tests/test_oracle_awq.py",
    "awq_ties_away": "tests/test_oracle_awq.py",
    "gelu_erf_form": "tests/test_oracle_mlp_pair.py",
    "mlp_unfused_not_rounded": "tests/test_oracle_mlp_pair.py",
}

MUTATIONS = ["ties_away_from_zero", "bias_dropped", "branch_sign", "tensor_scale_divisor", "lambda_inverted",
             "no_sign_convention", "e4m3_two_mantissa_bits", "e4m3_max_240", "bf16_smoothed_activations",
             "alpha_without_s_w", "s_x_unsmoothed", "nibble_order", "no_zero_guard", "unbalanced_split"]


def apply_from_env():
    import os

    name = os.environ.get("SVDQ_ORACLE_MUTATION")
    if name:
        from oracle import svdq_oracle as O

        _apply(O, name)
