"""Parity of the awq_w4a16 path (int4 weight quantizer and the 4-bit-weight GEMV for the
modulation projections, "Nunchaku Lite in Diffusers", kernel families) with the fp64 oracle,
through the C ABI.

Bit-exact: codes, fp16 scales and zero points of the quantizer (both sides decide in fp32).
Within tolerance: the GEMV output, max |Y - Y_ref| / max(|Y_ref|, 1e-2 rms(Y_ref)) <= 1e-2
against the oracle's fp64 product of the dequantized weights (the layer output's bound).
"""
import numpy as np
import pytest

from oracle import svdq_oracle as O
from synth import bf16_bits_to_f32, make_modulation_inputs
from tests.awq_layout import tile_layout
from tests.gpu_helpers import Y_TOL, bf16_tensor_to_np, rel_err_floor, x_to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def lib():
    from bit_rank_compensated_b200 import svdq

    svdq.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return svdq


def _special_rows(W):
    W = W.copy()
    W[0, :64] = 0.0                   # zero group: range raised to 1e-5
    W[1, 64:128] = 0.25               # constant positive group: codes saturate at 15
    W[2, :64] += 0.5                  # shifted group: zero point clamps at 0
    s = 2.0 ** -7                     # a group on the grid (lossless), with ties to even
    W[3, :64] = ((np.arange(64) % 16) - 5) * s
    W[3, 2:6] = np.array([0.5, 1.5, -2.5, 3.5]) * s
    return W


@pytest.mark.parametrize("N,K", [(300, 640), (37, 64), (64, 3072)])
def test_quantizer_bit_exact(lib, N, K):
    _, W, _ = make_modulation_inputs(1, K, N, seed=N)
    W = _special_rows(W)
    wq, sc, zp = lib.awq_quantize_weights(torch.from_numpy(W).cuda())
    torch.cuda.synchronize()
    q, s, z = O.awq_quantize(W)
    np.testing.assert_array_equal(wq.cpu().numpy(), O.pack_codes(q))
    np.testing.assert_array_equal(sc.cpu().numpy().astype(np.float64), s)
    np.testing.assert_array_equal(zp.cpu().numpy(), z)


@pytest.mark.parametrize("N,K", [(37, 128), (300, 640)])
def test_pack_layout(lib, N, K):
    _, W, _ = make_modulation_inputs(1, K, N, seed=N + 1)
    q, s, z = O.awq_quantize(W)
    wt, szt = lib.awq_pack_weights(torch.from_numpy(O.pack_codes(q)).cuda(),
                                   torch.from_numpy(s.astype(np.float16)).cuda(), torch.from_numpy(z).cuda())
    torch.cuda.synchronize()
    want_wt, want_sz = tile_layout(q, s, z)
    np.testing.assert_array_equal(wt.cpu().numpy(), want_wt)
    np.testing.assert_array_equal(szt.cpu().numpy(), want_sz)


def _oracle_linear(lib, M, N, K, seed, with_bias=True):
    Xb, W, b = make_modulation_inputs(M, K, N, seed=seed)
    q, s, z = O.awq_quantize(W)
    lin = lib.AwqLinear(torch.from_numpy(O.pack_codes(q)).cuda(), torch.from_numpy(s.astype(np.float16)).cuda(),
                        torch.from_numpy(z).cuda(), torch.from_numpy(b).cuda() if with_bias else None)
    Y_ref = O.awq_linear(bf16_bits_to_f32(Xb).astype(np.float64), q, s, z, b if with_bias else None)
    return Xb, lin, Y_ref


# K = 128 and 256 give 2 and 4 groups per row, so 2 and 4 warps share a row block (the other
# shapes use 1 or 8)
# The launch shape (warps, tiles in flight, warps per row block, groups per step) depends on K and
# N; these cover every compiled (ring slots, groups per step) pair: (4,4) (2,4) (8,2) (2,2) (4,2)
# (16,1) (8,1) (4,1) (2,1), and odd group counts per slice.
@pytest.mark.parametrize("M,N,K", [(1, 18432, 3072), (2, 9216, 3072), (3, 333, 576), (5, 64, 1024), (8, 130, 6144),
                                   (1, 1, 64), (7, 4100, 12288), (1, 1000, 128), (2, 1000, 256), (1, 24000, 4224),
                                   (1, 96, 4160), (1, 500, 10560), (2, 300, 11840)])
def test_gemv_matches_oracle(lib, M, N, K):
    Xb, lin, Y_ref = _oracle_linear(lib, M, N, K, seed=M, with_bias=M != 5)
    Y = lib.awq_gemv_w4a16(x_to_device(Xb), lin)
    torch.cuda.synchronize()
    assert rel_err_floor(bf16_tensor_to_np(Y).reshape(Y_ref.shape), Y_ref) <= Y_TOL


def test_gemv_repeats_bit_for_bit(lib):
    # fixed reduction order (slices summed in order): two launches give identical bits
    Xb, lin, _ = _oracle_linear(lib, 2, 2048, 3072, seed=9)
    X = x_to_device(Xb)
    Y1 = lib.awq_gemv_w4a16(X, lin).clone()
    Y2 = lib.awq_gemv_w4a16(X, lin)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


def test_quantize_then_gemv(lib):
    # the library's own quantizer feeding its GEMV: FLUX double-block modulation (6 x 3072 outputs)
    M, K, N = 1, 3072, 18432
    Xb, W, b = make_modulation_inputs(M, K, N, seed=7)
    lin = lib.AwqLinear.from_float(torch.from_numpy(W).cuda(), torch.from_numpy(b).cuda())
    Y = lib.awq_gemv_w4a16(x_to_device(Xb), lin)
    torch.cuda.synchronize()
    q, s, z = O.awq_quantize(W)
    Y_ref = O.awq_linear(bf16_bits_to_f32(Xb).astype(np.float64), q, s, z, b)
    assert rel_err_floor(bf16_tensor_to_np(Y).reshape(Y_ref.shape), Y_ref) <= Y_TOL


def test_rejects_unsupported_shapes(lib):
    Xb, W, b = make_modulation_inputs(9, 128, 16)
    lin = lib.AwqLinear.from_float(torch.from_numpy(W).cuda())
    with pytest.raises(lib.SvdqError):
        lib.awq_gemv_w4a16(x_to_device(Xb), lin)  # 9 tokens
    with pytest.raises(lib.SvdqError):
        lib.awq_quantize_weights(torch.zeros(4, 96, device="cuda"))  # K % 64
    with pytest.raises(lib.SvdqError):
        big = lib.AwqLinear.from_float(torch.zeros(16, 16384, device="cuda"))  # K above 12288
        lib.awq_gemv_w4a16(torch.zeros(1, 16384, dtype=torch.bfloat16, device="cuda"), big)
    torch.cuda.synchronize()
