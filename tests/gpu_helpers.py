"""Helpers for the GPU parity tests: move oracle-prepared layers and synthetic inputs to the
device and compare GPU outputs with the oracle's.

Direction of data: the oracle and the generators produce inputs and expected values; the
CUDA library only ever receives them as inputs. Nothing computed by the library is fed back
into the oracle.
"""
from __future__ import annotations

import numpy as np

from oracle import svdq_oracle as O
from synth import bf16_bits_to_f32, f32_to_bf16_bits
from tests import svdq_formats as F

# Output tolerance: max_i |Y_i - Y_ref_i| / max(|Y_ref_i|, tau) <= 1e-2 with the floor
# tau = 1e-2 * rms(Y_ref) (keeps entries near zero from dominating).
Y_TOL = 1e-2
Y_FLOOR = 1e-2


def rel_err_floor(got, ref, floor=Y_FLOOR):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    tau = floor * np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(got - ref) / np.maximum(np.abs(ref), tau)))


def fro_rel(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


def oracle_layer_arrays(layer: O.Layer):
    """Packs an oracle layer into the library's storage formats (host numpy arrays)."""
    N, K, r = layer.N, layer.K, layer.rank
    wq = O.pack_codes(layer.w_codes)
    ws = F.scales_to_blocked(layer.w_scales, (N + 255) // 256 * 256)
    L1t = f32_to_bf16_bits(layer.L1.T.astype(np.float32)) if r else None
    L2t = f32_to_bf16_bits(layer.L2.T.astype(np.float32)) if r else None
    return dict(N=N, K=K, rank=r, wq=wq, ws=ws, inv_lambda=layer.inv_lam.astype(np.float32), L1t=L1t, L2t=L2t,
                bias=layer.bias.astype(np.float32), s_w=layer.s_w, s_x=layer.s_x, lam=layer.lam.astype(np.float32))


def to_device_layer(layer: O.Layer):
    from bit_rank_compensated_b200 import svdq

    return svdq.Layer.from_arrays(**oracle_layer_arrays(layer))


def x_to_device(Xb):
    import torch

    return torch.from_numpy(np.ascontiguousarray(Xb).view(np.int16)).cuda().view(torch.bfloat16)


def bf16_tensor_to_np(t):
    import torch

    return bf16_bits_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)


def alpha32(layer: O.Layer) -> float:
    return float(np.float32(np.float32(layer.s_x) * np.float32(layer.s_w)))


def lora_pair_bits(v):
    """[hi | lo] bf16 planes of fp32 values v (rows x r): hi = bf16(v), lo = bf16(v - hi)."""
    v32 = np.asarray(v, dtype=np.float32)
    hi = f32_to_bf16_bits(v32)
    lo = f32_to_bf16_bits((v32 - bf16_bits_to_f32(hi)).astype(np.float32))
    return np.concatenate([hi, lo], axis=1)


def lora_pair_value(la_tensor, M, r):
    """hi + lo of a lora_act buffer, fp64 (M x r)."""
    both = bf16_tensor_to_np(la_tensor).reshape(M, 2 * r)
    return both[:, :r] + both[:, r:]
