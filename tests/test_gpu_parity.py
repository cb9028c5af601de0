"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Bit-exact: NVFP4 codes and e4m3 group scales of the activations (K1) and of the weights
(prepare / svdq_quantize_rows), the smoothing factors and the tensor scales.
Within tolerance (max |Y - Y_ref| / max(|Y_ref|, 1e-2 rms(Y_ref)) <= 1e-2): the layer output
and the pre-scaled down-projection lora_act.
"""
import numpy as np
import pytest

from oracle import svdq_oracle as O
from synth import CONFIGS, LayerShape, bf16_bits_to_f32, f32_to_bf16_bits, make_inputs
from tests import svdq_formats as F
from tests.gpu_helpers import (Y_TOL, alpha32, bf16_tensor_to_np, fro_rel, lora_pair_bits, lora_pair_value,
                               oracle_layer_arrays, rel_err_floor, to_device_layer, x_to_device)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def lib():
    from bit_rank_compensated_b200 import svdq

    svdq.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return svdq


def _problem(shape, M=None, seed=0):
    Xb, W, b, _ = make_inputs(shape, seed=seed, M=M)
    return Xb, bf16_bits_to_f32(Xb).astype(np.float64), W, b


def _shape(M, K, N, r, kind="spiky4"):
    return LayerShape(f"t{M}x{K}x{N}r{r}", M, K, N, r, kind)


def _k1_outputs(lib, Xb, layer_o):
    Ld = to_device_layer(layer_o)
    xq, xs, la = lib.quant_act_lora_down(x_to_device(Xb), Ld)
    torch.cuda.synchronize()
    return Ld, xq, xs, la


def _assert_k1_matches(Xb, X, layer_o, xq, xs, la):
    M, K = X.shape
    codes, scales, La = O.quant_act_lora_down(X, layer_o)
    np.testing.assert_array_equal(xq.cpu().numpy().reshape(M, K // 2), O.pack_codes(codes))
    xs_h = xs.cpu().numpy()
    Mp = (M + 127) // 128 * 128
    from bit_rank_compensated_b200 import svdq

    all_rows = svdq.unswizzle_scales(xs_h, Mp, K)
    np.testing.assert_array_equal(all_rows[:M], scales)
    assert not all_rows[M:].any(), "padding rows must carry zero scales"
    if layer_o.rank:
        # hi + lo carries the fp32 down-projection / alpha (fp32 tensor-core accumulation)
        got = lora_pair_value(la, M, layer_o.rank)
        assert rel_err_floor(got, La / alpha32(layer_o)) <= 1e-3
    return codes, scales, La


# ------------------------------------------------------------------ K2 layout pins
def _e2m1_vals(c):
    return O.e2m1_decode(c)


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (200, 272, 576), (1, 16, 64), (520, 320, 320)])
def test_k2_exact_on_power_of_two_scales(lib, M, N, K):
    # With power-of-two group scales, alpha = 1 and no bias every partial sum is exact in
    # fp32, so Y must equal bf16(exact dot product) bit for bit. Pins the operand and
    # scale-factor layouts of the block-scaled MMA.
    rng = np.random.default_rng(M + N + K)
    xc = rng.integers(0, 16, (M, K)).astype(np.uint8)
    wc = rng.integers(0, 16, (N, K)).astype(np.uint8)
    xc[xc == 8] = 0
    wc[wc == 8] = 0
    # scales in {1/2, 1, 2}: products are multiples of 2^-4 below 144, so sums over K <= 576
    # need at most 21 significant bits
    xsv = 2.0 ** rng.integers(-1, 2, (M, K // 16))
    wsv = 2.0 ** rng.integers(-1, 2, (N, K // 16))
    xs_codes = O.e4m3_encode(xsv)
    ws_codes = O.e4m3_encode(wsv)
    Xd = (_e2m1_vals(xc).reshape(M, K // 16, 16) * xsv[..., None]).reshape(M, K)
    Wd = (_e2m1_vals(wc).reshape(N, K // 16, 16) * wsv[..., None]).reshape(N, K)
    Y_exact = Xd @ Wd.T
    L = lib.Layer.from_arrays(N=N, K=K, rank=0, wq=O.pack_codes(wc), ws=F.scales_to_blocked(ws_codes, (N + 255) // 256 * 256),
                              inv_lambda=np.ones(K, np.float32), L1t=None, L2t=None, bias=None, s_w=1.0, s_x=1.0)
    xq = torch.from_numpy(O.pack_codes(xc).reshape(-1)).cuda()
    xs = torch.from_numpy(F.scales_to_blocked(xs_codes, (M + 127) // 128 * 128)).cuda()
    Y = lib.gemm_w4a4_lora_up(xq, xs, None, M, L)
    torch.cuda.synchronize()
    got = Y.view(torch.int16).cpu().numpy().view(np.uint16)
    want = f32_to_bf16_bits(Y_exact.astype(np.float32))
    np.testing.assert_array_equal(got, want)
    assert lib.last_device_error() == 0


@pytest.mark.parametrize("rank", [16, 32, 64, 128])
def test_k2_exact_low_rank_branch(lib, rank):
    # Small integers in lora_act and L2 with all 4-bit codes zero: Y = bf16(lora_act L2 + bias)
    # exactly (alpha = 1). Pins the bf16 operand layouts for every swizzle width.
    M, N, K = 130, 272, 128
    rng = np.random.default_rng(rank)
    la = rng.integers(-4, 5, (M, rank)).astype(np.float32)
    L2 = rng.integers(-4, 5, (rank, N)).astype(np.float32)
    bias = rng.integers(-8, 9, N).astype(np.float32)
    L = lib.Layer.from_arrays(N=N, K=K, rank=rank, wq=np.zeros((N, K // 2), np.uint8),
                              ws=np.zeros((N + 255) // 256 * 256 * K // 16, np.uint8), inv_lambda=np.ones(K, np.float32),
                              L1t=np.zeros((rank, K), np.uint16), L2t=f32_to_bf16_bits(L2.T.copy()), bias=bias,
                              s_w=1.0, s_x=1.0)
    xq = torch.zeros(M * K // 2, dtype=torch.uint8, device="cuda")
    xs = torch.zeros((M + 127) // 128 * 128 * K // 16, dtype=torch.uint8, device="cuda")
    lat = torch.from_numpy(lora_pair_bits(la).view(np.int16)).cuda().view(torch.bfloat16)
    Y = lib.gemm_w4a4_lora_up(xq, xs, lat, M, L)
    torch.cuda.synchronize()
    want = f32_to_bf16_bits((la.astype(np.float64) @ L2 + bias).astype(np.float32))
    np.testing.assert_array_equal(Y.view(torch.int16).cpu().numpy().view(np.uint16), want)


# ------------------------------------------------------------------ K1
def test_k1_tiny_bit_exact(lib):
    Xb, X, W, b = _problem(CONFIGS["tiny"])
    layer_o = O.prepare(W, b, O.calibration_absmax(X), 16)
    _, xq, xs, la = _k1_outputs(lib, Xb, layer_o)
    _assert_k1_matches(Xb, X, layer_o, xq, xs, la)
    assert lib.last_device_error() == 0


@pytest.mark.parametrize("M,K,N,r", [(1, 64, 16, 16), (129, 576, 272, 32), (300, 1024, 640, 64), (77, 768, 256, 128),
                                     (513, 512, 512, 0)])
def test_k1_ragged_shapes_bit_exact(lib, M, K, N, r):
    Xb, X, W, b = _problem(_shape(M, K, N, r), seed=1)
    layer_o = O.prepare(W, b, O.calibration_absmax(X), r)
    _, xq, xs, la = _k1_outputs(lib, Xb, layer_o)
    _assert_k1_matches(Xb, X, layer_o, xq, xs, la)


def test_k1_is_deterministic(lib):
    Xb, X, W, b = _problem(_shape(600, 3072, 256, 32), seed=2)
    layer_o = O.prepare(W, b, O.calibration_absmax(X), 32)
    Ld = to_device_layer(layer_o)
    Xd = x_to_device(Xb)
    first = [t.clone() for t in lib.quant_act_lora_down(Xd, Ld)]
    for _ in range(3):
        again = lib.quant_act_lora_down(Xd, Ld)
        for a, c in zip(first, again):
            assert torch.equal(a.view(torch.uint8), c.view(torch.uint8))


# ------------------------------------------------------------------ K1 + K2 vs oracle
@pytest.mark.parametrize("rank", [0, 16, 32, 64, 128])
def test_layer_rank_sweep(lib, rank):
    Xb, X, W, b = _problem(_shape(300, 1024, 640, rank), seed=3)
    layer_o = O.prepare(W, b, O.calibration_absmax(X), rank)
    Ld, xq, xs, la = _k1_outputs(lib, Xb, layer_o)
    codes, scales, La = _assert_k1_matches(Xb, X, layer_o, xq, xs, la)
    Y = lib.gemm_w4a4_lora_up(xq, xs, la, X.shape[0], Ld)
    torch.cuda.synchronize()
    Y_ref = O.gemm_w4a4_lora_up(codes, scales, La, layer_o)
    got = bf16_tensor_to_np(Y).reshape(Y_ref.shape)
    assert rel_err_floor(got, Y_ref) <= Y_TOL
    assert fro_rel(got, Y_ref) <= 5e-3
    assert lib.last_device_error() == 0


def test_k2_fed_oracle_activations(lib):
    # K2 alone, on the oracle's codes / scales / down-projection (as a hi/lo pair of La / alpha).
    Xb, X, W, b = _problem(CONFIGS["tiny"])
    layer_o = O.prepare(W, b, O.calibration_absmax(X), 16)
    Ld = to_device_layer(layer_o)
    codes, scales, La = O.quant_act_lora_down(X, layer_o)
    M, K = X.shape
    xq = torch.from_numpy(O.pack_codes(codes).reshape(-1)).cuda()
    xs = torch.from_numpy(F.scales_to_blocked(scales, (M + 127) // 128 * 128)).cuda()
    la = torch.from_numpy(lora_pair_bits(La / alpha32(layer_o)).view(np.int16)).cuda()
    Y = lib.gemm_w4a4_lora_up(xq, xs, la.view(torch.bfloat16), M, Ld)
    torch.cuda.synchronize()
    Y_ref = O.gemm_w4a4_lora_up(codes, scales, La, layer_o)
    assert rel_err_floor(bf16_tensor_to_np(Y).reshape(Y_ref.shape), Y_ref) <= Y_TOL


def test_unfused_baseline_matches_oracle(lib):
    Xb, X, W, b = _problem(_shape(260, 1024, 512, 32), seed=4)
    layer_o = O.prepare(W, b, O.calibration_absmax(X), 32)
    Ld = to_device_layer(layer_o)
    M = X.shape[0]
    bufs = lib.alloc_activations(M, Ld)
    Y = torch.empty(M, Ld.N, dtype=torch.bfloat16, device="cuda")
    lib.unfused_forward(x_to_device(Xb), Ld, bufs, Y)
    torch.cuda.synchronize()
    xq, xs, la = bufs
    _assert_k1_matches(Xb, X, layer_o, xq, xs, la)
    Y_ref = O.layer_forward(X, layer_o)
    # The unfused branch writes the 4-bit GEMM's output as bf16 and the up-projection reads it
    # back (the extra 16-bit output round trip), so each element carries one more bf16
    # rounding of the intermediate Y_mid = alpha * (4-bit product) + b. With the bf16 unit
    # roundoff 2^-8 the bound is 2^-8 (|Y_mid| + |Y|) plus fp32 accumulation noise.
    codes, scales, La = O.quant_act_lora_down(X, layer_o)
    Y_mid = O.gemm_w4a4_lora_up(codes, scales, La[:, :0], O.Layer(**{**layer_o.__dict__, "rank": 0}))
    got = bf16_tensor_to_np(Y).reshape(Y_ref.shape)
    bound = 2.0 ** -8 * (np.abs(Y_mid) + np.abs(Y_ref)) * 1.01 + 1e-4 * np.sqrt(np.mean(Y_ref ** 2))
    assert np.all(np.abs(got - Y_ref) <= bound)
    assert fro_rel(got, Y_ref) <= 5e-3


def test_forward_host_buffers(lib):
    Xb, X, W, b = _problem(CONFIGS["tiny"])
    layer_o = O.prepare(W, b, O.calibration_absmax(X), 16)
    Ld = to_device_layer(layer_o)
    M = X.shape[0]
    Xh = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).pin_memory()
    Yh = torch.empty(M, Ld.N, dtype=torch.bfloat16).pin_memory()
    Xd = torch.empty(M, Ld.K, dtype=torch.bfloat16, device="cuda")
    Yd = torch.empty(M, Ld.N, dtype=torch.bfloat16, device="cuda")
    lib.linear_forward_host(Xh, Ld, Xd, lib.alloc_activations(M, Ld), Yd, Yh)
    Y_ref = O.layer_forward(X, layer_o)
    assert rel_err_floor(bf16_tensor_to_np(Yh).reshape(Y_ref.shape), Y_ref) <= Y_TOL


@pytest.mark.parametrize("M,rank", [(300, 32), (1100, 16), (1024, 0), (1, 32)])
def test_forward_host_buffers_chunked(lib, M, rank):
    # the host-buffer path runs in row chunks of multiples of 256 rows (copies overlapping the
    # kernels of the neighbouring chunks): the output must be the whole-M device call's, bit for
    # bit, from pinned and from pageable host buffers
    Xb, X, W, b = _problem(_shape(M, 768, 512, rank), seed=M)
    layer_o = O.prepare(W, b, O.calibration_absmax(X), rank)
    Ld = to_device_layer(layer_o)
    Xd0 = x_to_device(Xb)
    Y_dev = lib.linear_forward(Xd0, Ld)
    torch.cuda.synchronize()
    want = Y_dev.view(torch.int16).cpu().numpy()
    for pinned in (True, False):
        Xh = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16)
        Yh = torch.empty(M, Ld.N, dtype=torch.bfloat16)
        if pinned:
            Xh, Yh = Xh.pin_memory(), Yh.pin_memory()
        Xd = torch.empty(M, Ld.K, dtype=torch.bfloat16, device="cuda")
        Yd = torch.empty(M, Ld.N, dtype=torch.bfloat16, device="cuda")
        lib.linear_forward_host(Xh, Ld, Xd, lib.alloc_activations(M, Ld), Yd, Yh)
        np.testing.assert_array_equal(Yh.view(torch.int16).numpy(), want)
    assert lib.last_device_error() == 0


# ------------------------------------------------------------------ prepare
def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("M,K,N,r", [(256, 512, 512, 16), (192, 1024, 384, 32), (128, 768, 256, 64), (64, 256, 128, 0)])
def test_prepare_matches_oracle(lib, M, K, N, r):
    Xb, X, W, b = _problem(_shape(M, K, N, r), seed=5)
    layer_o = O.prepare(W, b, O.calibration_absmax(X), r)
    ax = lib.act_absmax(x_to_device(Xb))
    np.testing.assert_array_equal(ax.cpu().numpy(), O.calibration_absmax(X).astype(np.float32))
    Ld = lib.prepare_weights(torch.from_numpy(W).cuda(), torch.from_numpy(b).cuda(), ax, r)
    np.testing.assert_array_equal(Ld.lam.cpu().numpy(), layer_o.lam.astype(np.float32))
    np.testing.assert_array_equal(Ld.inv_lambda.cpu().numpy(), layer_o.inv_lam.astype(np.float32))
    assert Ld.s_x == np.float32(layer_o.s_x)
    ref = oracle_layer_arrays(layer_o)
    if r:
        # Two independent fp64 SVD routes agree to ~1e-13, far below a bf16 step, so the
        # rounded factors agree bit for bit.
        np.testing.assert_array_equal(_bits(Ld.L1t).reshape(r, K), ref["L1t"])
        np.testing.assert_array_equal(_bits(Ld.L2t).reshape(N, r), ref["L2t"])
    assert Ld.s_w == np.float32(layer_o.s_w)
    np.testing.assert_array_equal(Ld.wq.cpu().numpy().reshape(N, K // 2), ref["wq"])
    np.testing.assert_array_equal(Ld.ws.cpu().numpy(), ref["ws"])


def test_quantize_rows_bit_exact(lib):
    # The weight quantizer on the oracle's fp32 residual.
    Xb, X, W, b = _problem(CONFIGS["tiny"])
    layer_o = O.prepare(W, b, O.calibration_absmax(X), 16)
    R = torch.from_numpy(np.ascontiguousarray(layer_o.R.astype(np.float32))).cuda()
    codes, scales = lib.quantize_rows(R, layer_o.s_w, 256)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes.cpu().numpy().reshape(layer_o.N, -1), O.pack_codes(layer_o.w_codes))
    np.testing.assert_array_equal(scales.cpu().numpy(), F.scales_to_blocked(layer_o.w_scales, 512))


def test_quantize_rows_ties_and_lossless(lib):
    # Exact e2m1 ties and lossless grid values through the hardware conversions.
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    rows = [np.concatenate([[6.0], np.tile(grid, 2)[:15]]) * 2.0 ** k for k in range(-4, 5)]
    ties = np.array([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, -0.1])
    rows.append(ties)
    A = np.stack([np.concatenate([r, -r, r * 0.5, r]) for r in rows]).astype(np.float32)
    s = 1.0
    codes, scales = lib.quantize_rows(torch.from_numpy(A).cuda(), s, 128)
    torch.cuda.synchronize()
    wc, wsc = O.nvfp4_quantize(A.astype(np.float64), s)
    np.testing.assert_array_equal(codes.cpu().numpy().reshape(A.shape[0], -1), O.pack_codes(wc))
    np.testing.assert_array_equal(lib.unswizzle_scales(scales.cpu().numpy(), A.shape[0], A.shape[1]), wsc)


def test_prepare_then_forward_tiny(lib):
    Xb, X, W, b = _problem(CONFIGS["tiny"])
    Xd = x_to_device(Xb)
    Ld = lib.prepare_weights(torch.from_numpy(W).cuda(), torch.from_numpy(b).cuda(), lib.act_absmax(Xd), 16)
    Y = lib.linear_forward(Xd, Ld)
    torch.cuda.synchronize()
    Y_ref = O.layer_forward(X, O.prepare(W, b, O.calibration_absmax(X), 16))
    assert rel_err_floor(bf16_tensor_to_np(Y).reshape(Y_ref.shape), Y_ref) <= Y_TOL


# ------------------------------------------------------------------ errors
def test_invalid_arguments_are_rejected(lib):
    Xb, X, W, b = _problem(CONFIGS["tiny"])
    layer_o = O.prepare(W, b, O.calibration_absmax(X), 16)
    Ld = to_device_layer(layer_o)
    Xd = x_to_device(Xb)
    # Only cases that the host rejects before any launch.
    Ld.s.K = 500  # K % 64 != 0
    with pytest.raises(lib.SvdqError) as e:
        lib.quant_act_lora_down(Xd, Ld)
    assert e.value.status == 1
    Ld.s.K = 512
    Ld.s.rank = 24
    with pytest.raises(lib.SvdqError) as e:
        lib.quant_act_lora_down(Xd, Ld)
    assert e.value.status == 1
    Ld.s.rank = 16
    bad = torch.empty(256 * 512 + 8, dtype=torch.bfloat16, device="cuda")[1:1 + 256 * 512].view(256, 512)
    with pytest.raises(lib.SvdqError) as e:
        lib.quant_act_lora_down(bad, Ld)
    assert e.value.status == 3


def test_quantize_rows_near_ties(lib):
    # Quotients within a few ulps of every e2m1 rounding threshold, with a group scale
    # (1.125) whose reciprocal is inexact: exercises the exact-division fallback.
    rng = np.random.default_rng(11)
    t = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    rows = []
    for _ in range(64):
        g = np.empty(16)
        g[0] = 6.75  # amax = 6 * 1.125 -> group scale 1.125 at s = 1
        k = rng.integers(-24, 25, 15)
        tt = rng.choice(t, 15) * rng.choice([-1.0, 1.0], 15)
        g[1:] = (np.float32(tt * 1.125) * (1.0 + k * 2.0 ** -23)).astype(np.float32)
        rows.append(g)
    A = np.stack(rows).reshape(16, 64).astype(np.float32)
    codes, scales = lib.quantize_rows(torch.from_numpy(A).cuda(), 1.0, 128)
    torch.cuda.synchronize()
    wc, wsc = O.nvfp4_quantize(A.astype(np.float64), 1.0)
    np.testing.assert_array_equal(codes.cpu().numpy().reshape(A.shape[0], -1), O.pack_codes(wc))
    np.testing.assert_array_equal(lib.unswizzle_scales(scales.cpu().numpy(), A.shape[0], 64), wsc)


@pytest.mark.parametrize("rank", [0, 32])
def test_k1_near_ties_take_the_exact_path(lib, rank):
    # Smoothed activations whose quotients by the group scale sit on, or within a few ulps of,
    # every e2m1 rounding threshold; the scale 1.125 has an inexact reciprocal. The bracket ends
    # disagree for nearly every group, so the activation kernel's correctly rounded fallback
    # decides the codes (ties to even included).
    rng = np.random.default_rng(12)
    M, K, N = 200, 512, 128
    t = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    X = rng.choice(t, (M, K)) * 1.125 * rng.choice([-1.0, 1.0], (M, K))
    X[:, ::16] = 6.75 * rng.choice([-1.0, 1.0], (M, K // 16))  # group amax: scale 1.125 at s_x = 1
    il = (1.0 + rng.integers(-6, 7, K) * 2.0 ** -23).astype(np.float32)
    il[::16] = 1.0
    Xb = f32_to_bf16_bits(X.astype(np.float32))
    assert np.array_equal(bf16_bits_to_f32(Xb).astype(np.float64), X)  # the values are bf16-exact
    Ld = lib.Layer.from_arrays(N=N, K=K, rank=rank, wq=np.zeros((N, K // 2), np.uint8),
                               ws=np.zeros(lib.weight_scale_bytes(N, K), np.uint8), inv_lambda=il,
                               L1t=np.zeros((rank, K), np.uint16) if rank else None,
                               L2t=np.zeros((N, rank), np.uint16) if rank else None, bias=None, s_w=1.0, s_x=1.0)
    xq, xs, _ = lib.quant_act_lora_down(x_to_device(Xb), Ld)
    torch.cuda.synchronize()
    codes, scales = O.nvfp4_quantize(O.f32(X * il.astype(np.float64)[None, :]), 1.0)
    np.testing.assert_array_equal(xq.cpu().numpy().reshape(M, K // 2), O.pack_codes(codes))
    Mp = (M + 127) // 128 * 128
    np.testing.assert_array_equal(lib.unswizzle_scales(xs.cpu().numpy(), M, K), scales)
    assert lib.last_device_error() == 0


def test_bounded_wait_gives_up_and_context_survives(lib):
    # The bounded waits every kernel uses, against an mbarrier nothing signals, with a 2 ms
    # limit: the wait gives up, records the timeout (kernel id 5, site 1) and the kernel
    # returns; the context stays usable for the next layer call.
    import time
    t0 = time.perf_counter()
    lib.selftest_wait_timeout(2000)
    code = lib.last_device_error()
    assert time.perf_counter() - t0 < 5.0
    assert code == (5 << 16) | (1 << 8) | 1
    assert lib.last_device_error() == 0  # read clears the word
    Xb, X, W, b = _problem(CONFIGS["tiny"])
    layer_o = O.prepare(W, b, O.calibration_absmax(X), 16)
    _, xq, xs, la = _k1_outputs(lib, Xb, layer_o)
    _assert_k1_matches(Xb, X, layer_o, xq, xs, la)
    assert lib.last_device_error() == 0
