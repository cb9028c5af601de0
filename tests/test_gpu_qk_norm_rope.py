"""Parity of the fused QKV output stage (K2 with per-head Q/K RMS normalization and rotary
embedding, "Nunchaku Lite in Diffusers", section on structural rewrites) and of its unfused
baseline with the fp64 oracle, through the C ABI.

Tolerance of the fused path: per section (Q, K, V), max |Z - Z_ref| / max(|Z_ref|, 1e-2
rms(Z_ref)) <= 1e-2, the layer output's bound; the normalization reads the fp32 values, so the
only 16-bit rounding is the final one. The unfused step reads the projection's bf16 output
back, which adds one rounding before the normalization; its bound is derived below.
"""
import numpy as np
import pytest

from oracle import svdq_oracle as O
from synth import CONFIGS, LayerShape, bf16_bits_to_f32, make_inputs, qk_norm_weights, rope_table
from tests.gpu_helpers import Y_TOL, bf16_tensor_to_np, rel_err_floor, to_device_layer, x_to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
D = 128
EPS = 1e-6


@pytest.fixture(scope="module")
def lib():
    from bit_rank_compensated_b200 import svdq

    svdq.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return svdq


def _case(M, heads, K, rank, seed=0, n_text=None):
    shape = LayerShape(f"qkv{M}x{K}h{heads}r{rank}", M, K, 3 * heads * D, rank, "spiky1pct")
    Xb, W, b, _ = make_inputs(shape, seed=seed)
    X = bf16_bits_to_f32(Xb).astype(np.float64)
    layer_o = O.prepare(W, b, O.calibration_absmax(X), rank)
    table = rope_table(M, D, n_text=n_text)
    wq, wk = qk_norm_weights(D, seed)
    return Xb, X, layer_o, table, wq, wk


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _oracle_z(X, layer_o, table, wq, wk, heads, rows=None):
    Xr = X if rows is None else X[rows]
    codes, scales, La = O.quant_act_lora_down(Xr, layer_o)
    Y_ref = O.gemm_w4a4_lora_up(codes, scales, La, layer_o)
    t = table if rows is None else table[rows]
    c, s = t[..., 0].astype(np.float64), t[..., 1].astype(np.float64)
    Z = O.qk_norm_rope(Y_ref, heads, D, wq.astype(np.float64), wk.astype(np.float64), c, s, EPS)
    return Y_ref, Z


def _check_sections(got, ref, heads):
    w = heads * D
    for sec in range(3):
        g, r = got[:, sec * w:(sec + 1) * w], ref[:, sec * w:(sec + 1) * w]
        err = rel_err_floor(g, r)
        assert err <= Y_TOL, f"section {'QKV'[sec]}: {err:.3e}"


@pytest.mark.parametrize("M,heads,K,rank", [(256, 2, 512, 16), (200, 3, 576, 32), (129, 1, 256, 0), (300, 2, 1024, 64),
                                            (1, 1, 64, 16)])
def test_fused_stage_matches_oracle(lib, M, heads, K, rank):
    Xb, X, layer_o, table, wq, wk = _case(M, heads, K, rank, seed=M)
    Ld = to_device_layer(layer_o)
    xq, xs, la = lib.quant_act_lora_down(x_to_device(Xb), Ld)
    Z = lib.gemm_w4a4_lora_up_qk_norm_rope(xq, xs, la, M, Ld, heads, _dev(wq), _dev(wk), _dev(table), EPS)
    Y = lib.gemm_w4a4_lora_up(xq, xs, la, M, Ld)
    torch.cuda.synchronize()
    assert lib.last_device_error() == 0
    Y_ref, Z_ref = _oracle_z(X, layer_o, table, wq, wk, heads)
    got = bf16_tensor_to_np(Z).reshape(Z_ref.shape)
    _check_sections(got, Z_ref, heads)
    # V leaves the fused stage exactly as the plain output stage writes it
    w = heads * D
    np.testing.assert_array_equal(Z[:, 2 * w:].cpu().view(torch.int16).numpy(), Y[:, 2 * w:].cpu().view(torch.int16).numpy())


def test_unfused_step_matches_oracle(lib):
    M, heads = 260, 2
    Xb, X, layer_o, table, wq, wk = _case(M, heads, 512, 32, seed=5)
    Ld = to_device_layer(layer_o)
    xq, xs, la = lib.quant_act_lora_down(x_to_device(Xb), Ld)
    Y = lib.gemm_w4a4_lora_up(xq, xs, la, M, Ld)
    lib.qk_norm_rope(Y, heads, _dev(wq), _dev(wk), _dev(table), EPS)
    torch.cuda.synchronize()
    Y_ref, Z_ref = _oracle_z(X, layer_o, table, wq, wk, heads)
    got = bf16_tensor_to_np(Y).reshape(Z_ref.shape)
    w = heads * D
    # V: the plain projection's output
    assert rel_err_floor(got[:, 2 * w:], Z_ref[:, 2 * w:]) <= Y_TOL
    # Q, K: the step reads bf16(v); with bf16's unit roundoff 2^-8, |dv| <= 2^-8 |v|, which moves
    # each normalized value u by at most 2^-8 |u| directly and 2^-8 |u| through the mean square,
    # so |du| <= 2^-7 |u|; a rotation mixes the two values of a pair (|cos|, |sin| <= 1) and the
    # result is rounded to bf16 once more (2^-8 |z|). Margin 5% for the fp32 arithmetic.
    for sec, wv in ((0, wq), (1, wk)):
        blk = Y_ref[:, sec * w:(sec + 1) * w].reshape(M, heads, D)
        U = O.rms_norm_heads(blk, wv.astype(np.float64), EPS)
        pair = np.abs(U[..., 0::2]) + np.abs(U[..., 1::2])
        upair = np.repeat(pair, 2, axis=-1).reshape(M, w)
        z = Z_ref[:, sec * w:(sec + 1) * w]
        bound = 1.05 * (2.0 ** -7 * upair + 2.0 ** -8 * np.abs(z)) + 1e-6
        assert np.all(np.abs(got[:, sec * w:(sec + 1) * w] - z) <= bound)


def test_rejects_unsupported_shapes(lib):
    Xb, X, layer_o, table, wq, wk = _case(64, 1, 64, 16)
    Ld = to_device_layer(layer_o)
    xq, xs, la = lib.quant_act_lora_down(x_to_device(Xb), Ld)
    for heads, hd in ((2, 128), (1, 64)):
        with pytest.raises(lib.SvdqError):
            lib.gemm_w4a4_lora_up_qk_norm_rope(xq, xs, la, 64, Ld, heads, _dev(wq), _dev(wk), _dev(table), EPS,
                                               head_dim=hd)
    with pytest.raises(lib.SvdqError):
        lib.qk_norm_rope(torch.empty(4, 3 * 64, dtype=torch.bfloat16, device="cuda"), 1, _dev(wq), _dev(wk),
                         _dev(table), EPS, head_dim=64)
    torch.cuda.synchronize()


def test_qkv_full_size_sampled(lib):
    # The FLUX-like fused QKV workload (M = 4608 = 512 text + 4096 image tokens, 24 heads) in the
    # launch configuration the bench times: library prepare, K1, fused K2; 64 sampled rows
    # (text and image tokens) against the oracle.
    shape = CONFIGS["qkv"]
    heads = shape.N // (3 * D)
    Xb, W, b, _ = make_inputs(shape, seed=0)
    X = bf16_bits_to_f32(Xb).astype(np.float64)
    layer_o = O.prepare(W, b, O.calibration_absmax(X), shape.rank)
    table = rope_table(shape.M, D)
    wq, wk = qk_norm_weights(D, 0)
    Xd = x_to_device(Xb)
    Ld = lib.prepare_weights(torch.from_numpy(W).cuda(), torch.from_numpy(b).cuda(), lib.act_absmax(Xd), shape.rank)
    xq, xs, la = lib.quant_act_lora_down(Xd, Ld)
    Z = lib.gemm_w4a4_lora_up_qk_norm_rope(xq, xs, la, shape.M, Ld, heads, _dev(wq), _dev(wk), _dev(table), EPS)
    torch.cuda.synchronize()
    assert lib.last_device_error() == 0
    rows = np.sort(np.concatenate([np.random.default_rng(11).choice(512, 16, replace=False),
                                   512 + np.random.default_rng(12).choice(4096, 48, replace=False)]))
    _, Z_ref = _oracle_z(X, layer_o, table, wq, wk, heads, rows)
    got = bf16_tensor_to_np(Z[torch.from_numpy(rows).cuda()])
    _check_sections(got, Z_ref, heads)
