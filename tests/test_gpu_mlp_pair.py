"""Parity of the FLUX feed-forward pair (SVDQuant linear -> GELU -> SVDQuant linear) with the fp64 oracle.

"Nunchaku Lite in Diffusers", introduction of Nunchaku Lite (the engine's fused GELU / MLP kernels):
in the fused pair the up-projection's output stage computes h = GELU(alpha acc + b) in fp32 and
writes the down layer's NVFP4 activations and low-rank down-projection directly, so the intermediate
never reaches memory in 16 bits (oracle.mlp_pair(fused=True)). In the unfused pair the intermediate
is written as bf16 and read back (fused=False).

The down layer's activation codes are integers decided by floating point from h, and the kernel's
h (fp32 GEMM accumulation, fp32 GELU) differs from the oracle's fp64 h in the last bits. So:
  * codes and scales equal the oracle's everywhere except where the oracle's own value lies within
    a small interval (|dx| <= 1e-5 (|x| + group amax)) of a rounding threshold; there the kernel's
    code must be one of the codes that interval's ends round to (checked element by element), and
    such elements must be rare;
  * the down-projection (hi + lo) is within an element-wise bound derived from the arithmetic that
    separates the kernel's h from the oracle's (la_bound: the up layer's fp32 accumulation, GELU's
    slope, the hi / lo pair), and within 1e-4 of h L1s in Frobenius norm;
  * the pair's output Z is within the output tolerance of the oracle on every row whose codes and
    scales all equal the oracle's (the other rows are counted, and must be rare).
"""
import numpy as np
import pytest

from oracle import svdq_oracle as O
from synth import CONFIGS, LayerShape, bf16_bits_to_f32, make_inputs
from tests.gpu_helpers import (Y_TOL, alpha32, bf16_tensor_to_np, fro_rel, lora_pair_value, rel_err_floor,
                               to_device_layer, x_to_device)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

DELTA = 1e-5  # relative size of the interval of values the kernel's fp32 h may take


@pytest.fixture(scope="module")
def lib():
    from bit_rank_compensated_b200 import svdq

    svdq.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return svdq


def make_pair(M, K, N_up, N_d, r_u, r_d, seed=0):
    """Oracle-prepared up and down layers: X from the layer-normed MLP generator, the down layer
    calibrated on the oracle's fused intermediate H (its smoothing factors from max |H_j|)."""
    Xb, Wu, bu, _ = make_inputs(LayerShape("mlp_u", M, K, N_up, r_u, "layernorm1pct"), seed=seed)
    _, Wd, bd, _ = make_inputs(LayerShape("mlp_d", 1, N_up, N_d, r_d, "gelu_lognormal"), seed=seed + 1)
    X = bf16_bits_to_f32(Xb).astype(np.float64)
    up = O.prepare(Wu, bu, O.calibration_absmax(X), r_u)
    H = O.mlp_hidden(X, up, fused=True)
    down = O.prepare(Wd, bd, O.calibration_absmax(H), r_d)
    return Xb, X, up, down, H


def _e2m1_value_of(q):
    """Signed e2m1 value a quotient rounds to (oracle rounding)."""
    return O.e2m1_round(q)


def check_codes(xq_k, xs_k, H, down, delta=DELTA):
    """Element-wise validity of the kernel's codes / scales against the oracle's (see module doc).
    Returns (row mask of rows equal to the oracle everywhere, fraction of differing codes)."""
    M, Kd = H.shape
    G = Kd // 16
    Xh = O.f32(H * down.inv_lam[None, :])  # oracle's x_hat
    codes_o, scales_o = O.nvfp4_quantize(Xh, down.s_x)
    codes_k = O.unpack_codes(xq_k).reshape(M, Kd)
    same = (codes_k == codes_o)
    same_s = (xs_k == scales_o)
    row_equal = same.all(axis=1) & same_s.all(axis=1)
    # scales: the kernel's scale must lie between the codes of amax (1 -/+ 2 delta)
    Xg = Xh.reshape(M, G, 16)
    amax = np.abs(Xg).max(axis=2)
    d = O.f32(6.0 * down.s_x)
    s_lo = O.e4m3_encode(O.e4m3_round(O.f32(amax * (1 - 2 * delta) / d)))
    s_hi = O.e4m3_encode(O.e4m3_round(O.f32(amax * (1 + 2 * delta) / d)))
    bad_s = ~same_s & ((xs_k < s_lo) | (xs_k > s_hi))
    assert not bad_s.any(), f"{int(bad_s.sum())} scales outside their interval"
    # codes, with the kernel's own scale: value between the roundings of the interval's ends
    eff = O.f32(O.e4m3_decode(xs_k) * down.s_x)[..., None]
    e = delta * (np.abs(Xg) + amax[..., None])
    with np.errstate(divide="ignore", invalid="ignore"):
        lo = np.where(eff > 0, O.e2m1_round(O.f32((Xg - e) / eff)), 0.0)
        hi = np.where(eff > 0, O.e2m1_round(O.f32((Xg + e) / eff)), 0.0)
    vk = O.e2m1_decode(codes_k).reshape(M, G, 16)
    bad = ~same.reshape(M, G, 16) & ((vk < lo) | (vk > hi))
    assert not bad.any(), f"{int(bad.sum())} codes outside their interval"
    return row_equal, float(np.mean(~same))


def la_bound(X, up, down, H):
    """Element-wise bound on the fused down-projection's error against the oracle's fp64 value.
    The kernel's h differs from the oracle's through the up layer's fp32 accumulation: each
    v = s_x s_w sum_i q_x q_w + sum_j La_j L2_j + b is a sum of exactly represented terms, so its
    error is at most gamma sum |terms| with gamma = (K + r + 2) 2^-24 (fp32 summation of that many
    terms); GELU's slope is at most 1.13, and the 2^-16 relative error of the hi / lo pair and the
    fp32 accumulation of the sum over N_up inputs add 2^-15 |h| per term. So
    |dLa_j| <= sum_k (1.13 gamma T_k + 2^-15 |h_k|) |L1s_kj|, T_k the magnitude sum of v_k."""
    codes, scales, La_up = O.quant_act_lora_down(X, up)
    Xd = np.abs(O.nvfp4_dequantize(codes, scales))
    Wd = np.abs(O.nvfp4_dequantize(up.w_codes, up.w_scales))
    T = up.s_x * up.s_w * (Xd @ Wd.T) + np.abs(up.bias)[None, :]
    if up.rank:
        T = T + np.abs(La_up) @ np.abs(up.L2)
    gamma = (up.K + up.rank + 2) * 2.0 ** -24
    E = 1.13 * gamma * T + 2.0 ** -15 * np.abs(H)
    return E @ np.abs(down.L1) + 1e-30


def _run_fused(lib, Xb, up, down):
    M = Xb.shape[0]
    Lu, Ld = to_device_layer(up), to_device_layer(down)
    Xd = x_to_device(Xb)
    bufs = lib.alloc_activations(M, Lu)
    bufs_d = lib.alloc_activations(M, Ld)
    ws = lib.alloc_mlp_workspace(M, Lu, Ld)
    Z = torch.empty(M, Ld.N, dtype=torch.bfloat16, device="cuda")
    lib.mlp_forward(Xd, Lu, Ld, bufs, bufs_d, ws, Z)
    torch.cuda.synchronize()
    assert lib.last_device_error() == 0
    return bufs_d, Z


def _check_pair(lib, Xb, X, up, down, H, rows=None):
    M = X.shape[0]
    Kd = down.K
    (xq_d, xs_d, la_d), Z = _run_fused(lib, Xb, up, down)
    xq_k = xq_d.cpu().numpy().reshape(M, Kd // 2)
    Mp = (M + 127) // 128 * 128
    sc_all = lib.unswizzle_scales(xs_d.cpu().numpy(), Mp, Kd)
    assert not sc_all[M:].any(), "padding rows must carry zero scales"
    row_equal, frac = check_codes(xq_k, sc_all[:M], H, down)
    assert frac <= 1e-3, f"{frac:.2e} of the codes differ"
    assert row_equal.mean() >= 0.9, f"only {row_equal.mean():.3f} of the rows equal the oracle everywhere"
    codes_o, scales_o, La_o = O.quant_act_lora_down(H, down)
    if down.rank:
        got = lora_pair_value(la_d, M, down.rank) * alpha32(down)
        bound = la_bound(X, up, down, H)
        assert np.all(np.abs(got - La_o) <= bound), float(np.max(np.abs(got - La_o) / bound))
        assert fro_rel(got, La_o) <= 1e-4
    sel = np.arange(M) if rows is None else rows
    sel = sel[row_equal[sel]]
    Z_ref = O.gemm_w4a4_lora_up(codes_o[sel], scales_o[sel], La_o[sel], down)
    got = bf16_tensor_to_np(Z[torch.from_numpy(sel).cuda()])
    err = rel_err_floor(got, Z_ref)
    assert err <= Y_TOL, f"max floor-relative error {err:.3e} over {len(sel)} rows"
    # the whole output against the oracle's fused pair (rows with a code on a threshold included)
    Z_all_ref = O.gemm_w4a4_lora_up(codes_o, scales_o, La_o, down) if rows is None else None
    if Z_all_ref is not None:
        assert fro_rel(bf16_tensor_to_np(Z), Z_all_ref) <= 5e-3


@pytest.mark.parametrize("M,K,N_up,N_d,r_u,r_d", [
    (300, 512, 1024, 384, 32, 32),   # ragged M (a partial 256-row tile, padding scale rows)
    (129, 256, 576, 128, 16, 16),    # N_up not a multiple of 256 (half a tile past N)
    (256, 512, 768, 256, 0, 64),     # up layer without branch, down rank 64
    (200, 256, 512, 256, 128, 0),    # down layer without branch (no partials)
])
def test_fused_mlp_pair(lib, M, K, N_up, N_d, r_u, r_d):
    Xb, X, up, down, H = make_pair(M, K, N_up, N_d, r_u, r_d, seed=M)
    _check_pair(lib, Xb, X, up, down, H)


def test_fused_mlp_pair_is_deterministic(lib):
    Xb, X, up, down, H = make_pair(300, 512, 1024, 384, 32, 32, seed=5)
    (a_q, a_s, a_l), Za = _run_fused(lib, Xb, up, down)
    for _ in range(2):
        (b_q, b_s, b_l), Zb = _run_fused(lib, Xb, up, down)
        assert torch.equal(a_q, b_q) and torch.equal(a_s, b_s)
        assert torch.equal(a_l.view(torch.int16), b_l.view(torch.int16))
        assert torch.equal(Za.view(torch.int16), Zb.view(torch.int16))


def test_unfused_first_layer_gelu(lib):
    # The unfused pair's first layer writes bf16(GELU(alpha acc + b)). Against the oracle's
    # bf16(GELU(Y1)) (Y1 in fp64): GELU's slope is at most 1.13, so an output error within the
    # layer tolerance 1e-2 max(|Y1|, tau) moves h by at most 1.13 times that, plus the bf16
    # rounding of h (unit roundoff 2^-8).
    M, K, N = 300, 512, 1024
    Xb, X, up, down, H = make_pair(M, K, N, 256, 32, 32, seed=11)
    Lu = to_device_layer(up)
    xq, xs, la = lib.quant_act_lora_down(x_to_device(Xb), Lu)
    Hk = lib.gemm_w4a4_lora_up_gelu(xq, xs, la, M, Lu)
    torch.cuda.synchronize()
    Y1 = O.layer_forward(X, up)
    tau = 1e-2 * np.sqrt(np.mean(Y1 ** 2))
    H_ref = O.gelu_tanh(Y1)
    got = bf16_tensor_to_np(Hk).reshape(M, N)
    bound = 1.13 * 1e-2 * np.maximum(np.abs(Y1), tau) + 2.0 ** -8 * np.abs(H_ref) * 1.01
    assert np.all(np.abs(got - H_ref) <= bound)
    # and the rounding to bf16 happened after the GELU (the oracle's unfused intermediate)
    assert fro_rel(got, O.mlp_hidden(X, up, fused=False)) <= 5e-3


def test_fused_mlp_pair_rejects_bad_arguments(lib):
    Xb, X, up, down, H = make_pair(128, 256, 512, 128, 16, 16, seed=2)
    Lu, Ld = to_device_layer(up), to_device_layer(down)
    xq, xs, la = lib.quant_act_lora_down(x_to_device(Xb), Lu)
    ws = lib.alloc_mlp_workspace(128, Lu, Ld)
    small = ws[:16]
    with pytest.raises(lib.SvdqError) as e:
        lib.gemm_w4a4_lora_up_gelu_quant(xq, xs, la, 128, Lu, Ld, workspace=small)
    assert e.value.status == 1
    wrong = to_device_layer(O.prepare(np.zeros((128, 256), np.float32), None, np.ones(256), 16))
    with pytest.raises(lib.SvdqError) as e:  # down->K != up->N
        lib.gemm_w4a4_lora_up_gelu_quant(xq, xs, la, 128, Lu, wrong, workspace=ws)
    assert e.value.status == 1


def test_fused_mlp_pair_full_size(lib):
    # The FLUX feed-forward pair at the benchmark's size: M 4608, 3072 -> 12288 -> 3072, rank 32.
    up_s, down_s = CONFIGS["mlp_up"], CONFIGS["mlp_down"]
    Xb, Wu, bu, _ = make_inputs(up_s, seed=0)
    _, Wd, bd, _ = make_inputs(down_s, seed=0)
    X = bf16_bits_to_f32(Xb).astype(np.float64)
    up = O.prepare(Wu, bu, O.calibration_absmax(X), up_s.rank)
    H = O.mlp_hidden(X, up, fused=True)
    down = O.prepare(Wd, bd, O.calibration_absmax(H), down_s.rank)
    from tests.test_gpu_full_size import sample_rows

    _check_pair(lib, Xb, X, up, down, H, rows=sample_rows(X.shape[0]))
