"""Host-side behaviour of the C ABI, checked without a GPU: argument rejection (which comes
before any device query), the architecture refusal through the capability override hook, and
the pure-host scale unswizzling.

"Nunchaku Lite in Diffusers", hardware support ("دعم الأجهزة"): a GPU the kernels were not
built for gets a clear error, never wrong output. Nothing here launches a kernel: every call is
refused by the host checks, so the fake device addresses below are never dereferenced.
"""
import ctypes

import numpy as np
import pytest

from tests import svdq_formats as F

OK, INVALID, UNSUPPORTED, MISALIGNED = 0, 1, 2, 3
DEV = 0x7F0000000000  # a 16-byte aligned address that is never dereferenced (calls are refused first)
ODD = DEV + 8


@pytest.fixture(scope="module")
def lib():
    import os

    from bit_rank_compensated_b200 import build, svdq

    if not os.path.exists(svdq.LIB_PATH):
        build.build()
    return svdq.load()


@pytest.fixture
def unsupported(lib):
    """Capability override to an unsupported GPU for the duration of one test."""
    assert lib.svdq_test_override_capability(9, 0) == OK
    yield
    assert lib.svdq_test_override_capability(-1, 0) == OK


def _layer(N=512, K=512, rank=16, bias=True, wq=DEV):
    from bit_rank_compensated_b200.svdq import LayerStruct

    s = LayerStruct()
    s.N, s.K, s.rank, s.group = N, K, rank, 16
    s.w_tensor_scale, s.x_tensor_scale = 0.5, 0.25
    s.wq, s.ws, s.inv_lambda, s.lambda_ = wq, DEV, DEV, DEV
    s.L1t = DEV if rank else None
    s.L2t = DEV if rank else None
    s.bias = DEV if bias else None
    return s


def _p(v):
    return None if v is None else ctypes.c_void_p(v)


def _calls(lib, layer, X=DEV, M=256, out=DEV):
    """Every GPU entry point with otherwise valid arguments (fake device addresses)."""
    L = ctypes.byref(layer)
    P = _p
    N, K = layer.N, layer.K
    return {
        "svdq_act_absmax": lambda: lib.svdq_act_absmax(P(X), M, K, P(out), None),
        "svdq_quant_act_lora_down": lambda: lib.svdq_quant_act_lora_down(P(X), M, L, P(out), P(out), P(out), None),
        "svdq_gemm_w4a4_lora_up": lambda: lib.svdq_gemm_w4a4_lora_up(P(out), P(out), P(out), M, L, P(out), None),
        "svdq_linear_forward": lambda: lib.svdq_linear_forward(P(X), M, L, P(out), P(out), P(out), P(out), None),
        "svdq_linear_forward_host": lambda: lib.svdq_linear_forward_host(P(X), M, L, P(X), P(out), P(out), P(out),
                                                                         P(out), P(out), None),
        "svdq_baseline_lora_down": lambda: lib.svdq_baseline_lora_down(P(X), M, L, P(out), None),
        "svdq_baseline_quantize": lambda: lib.svdq_baseline_quantize(P(X), M, L, P(out), P(out), None),
        "svdq_baseline_gemm_w4a4": lambda: lib.svdq_baseline_gemm_w4a4(P(out), P(out), M, L, P(out), None),
        "svdq_baseline_lora_up": lambda: lib.svdq_baseline_lora_up(P(out), M, L, P(out), None),
        "svdq_quantize_rows": lambda: lib.svdq_quantize_rows(P(X), M, K, 1.0, 128, P(out), P(out), None),
        "svdq_gemm_w4a4_lora_up_qk_norm_rope": lambda: lib.svdq_gemm_w4a4_lora_up_qk_norm_rope(
            P(out), P(out), P(out), M, ctypes.byref(_layer(N=3 * 128, K=K, rank=layer.rank)), 1, 128, P(out),
            P(out), P(out), 1e-6, P(out), None),
        "svdq_qk_norm_rope": lambda: lib.svdq_qk_norm_rope(P(out), M, 1, 128, P(out), P(out), P(out), 1e-6, None),
        "svdq_awq_quantize_weights": lambda: lib.svdq_awq_quantize_weights(P(X), N, K, P(out), P(out), P(out), None),
        "svdq_awq_pack_weights": lambda: lib.svdq_awq_pack_weights(P(X), P(X), P(X), N, K, P(out), P(out), None),
        "svdq_awq_gemv_w4a16": lambda: lib.svdq_awq_gemv_w4a16(P(X), 1, P(X), P(X), None, N, K, P(out), None),
        "svdq_smoothing_factors_noalloc": lambda: lib.svdq_smoothing_factors_noalloc(
            P(X), P(X), N, K, P(out), P(out), P(out), None),
        "svdq_prepare_weights": lambda: lib.svdq_prepare_weights(P(X), None, P(X), N, K, layer.rank, L, P(out), 1 << 30,
                                                                 None),
        "svdq_gemm_w4a4_lora_up_gelu": lambda: lib.svdq_gemm_w4a4_lora_up_gelu(P(out), P(out), P(out), M, L, P(out),
                                                                               None),
        "svdq_gemm_w4a4_lora_up_gelu_quant": lambda: lib.svdq_gemm_w4a4_lora_up_gelu_quant(
            P(out), P(out), P(out), M, L, ctypes.byref(_layer(N=256, K=N, rank=16)), P(out), P(out), P(out), P(out),
            1 << 30, None),
        "svdq_mlp_forward": lambda: lib.svdq_mlp_forward(
            P(X), M, L, ctypes.byref(_layer(N=256, K=N, rank=16)), P(out), P(out), P(out), P(out), P(out), P(out),
            P(out), 1 << 30, P(out), None),
        "svdq_selftest_wait_timeout": lambda: lib.svdq_selftest_wait_timeout(1000, None),
        "svdq_last_device_error": lambda: lib.svdq_last_device_error(None, ctypes.byref(ctypes.c_uint32(0))),
    }


def test_every_gpu_entry_point_refuses_an_unsupported_gpu(lib, unsupported):
    for name, call in _calls(lib, _layer()).items():
        assert call() == UNSUPPORTED, name
    # also for another generation than the one below
    assert lib.svdq_test_override_capability(12, 0) == OK
    for name, call in _calls(lib, _layer()).items():
        assert call() == UNSUPPORTED, name


def test_refusal_names_the_required_gpu(lib):
    msg = lib.svdq_status_string(UNSUPPORTED).decode()
    assert "10.0" in msg and "B200" in msg


def test_override_hook_arguments(lib):
    assert lib.svdq_test_override_capability(100, 0) == INVALID
    assert lib.svdq_test_override_capability(9, 10) == INVALID
    assert lib.svdq_test_override_capability(-1, 0) == OK


def test_host_prepare_refuses_an_unsupported_gpu(lib, unsupported):
    W = np.zeros((256, 256), np.float32)
    ax = np.ones(256, np.float32)
    layer = _layer(N=256, K=256, rank=16)
    st = lib.svdq_prepare_weights_host(W.ctypes.data_as(ctypes.c_void_p), None, ax.ctypes.data_as(ctypes.c_void_p),
                                       256, 256, 16, ctypes.byref(layer), None, None)
    assert st == UNSUPPORTED


@pytest.mark.parametrize("case", ["N%16", "K%64", "rank", "M<=0", "M<0", "null X", "null layer wq", "null out",
                                  "s_x<=0", "s_x tiny", "s_w huge", "N<=0"])
def test_invalid_arguments_are_rejected_before_the_device(lib, unsupported, case):
    # The argument checks run before the capability check, so INVALID_ARG wins over the
    # (overridden) unsupported GPU: the rejection needs no device.
    layer = _layer()
    X, M, out = DEV, 256, DEV
    if case == "N%16":
        layer.N = 520
    elif case == "K%64":
        layer.K = 500
    elif case == "rank":
        layer.rank = 24
    elif case == "M<=0":
        M = 0
    elif case == "M<0":
        M = -5
    elif case == "null X":
        X = None
    elif case == "null layer wq":
        layer.wq = None
    elif case == "null out":
        out = None
    elif case == "s_x<=0":
        layer.x_tensor_scale = 0.0
    elif case == "s_x tiny":
        layer.x_tensor_scale = 2.0 ** -117  # below the range the exact quantizer covers
    elif case == "s_w huge":
        layer.w_tensor_scale = 2.0 ** 117
    elif case == "N<=0":
        layer.N = 0
    P = _p
    L = ctypes.byref(layer)
    assert lib.svdq_quant_act_lora_down(P(X), M, L, P(out), P(out), P(out), None) == INVALID
    if case != "null X":
        assert lib.svdq_gemm_w4a4_lora_up(P(out), P(out), P(out), M, L, P(out), None) == INVALID
    assert lib.svdq_linear_forward(P(X), M, L, P(out), P(out), P(out), P(out), None) == INVALID


def test_tensor_scale_range(lib, unsupported):
    # [2^-116, 2^116] is accepted (the call gets as far as the device check)
    for sx in (2.0 ** -116, 1.0, 2.0 ** 116):
        layer = _layer()
        layer.x_tensor_scale = sx
        assert lib.svdq_quant_act_lora_down(_p(DEV), 16, ctypes.byref(layer), _p(DEV), _p(DEV), _p(DEV),
                                            None) == UNSUPPORTED
    assert lib.svdq_quantize_rows(_p(DEV), 16, 64, 2.0 ** -117, 128, _p(DEV), _p(DEV), None) == INVALID
    assert lib.svdq_quantize_rows(_p(DEV), 16, 64, float("nan"), 128, _p(DEV), _p(DEV), None) == INVALID


def test_mlp_pair_shapes_are_checked_before_the_device(lib, unsupported):
    up = _layer(N=512, K=512, rank=16)
    P = _p
    for down in (_layer(N=256, K=256, rank=16),     # down K != up N
                 _layer(N=256, K=512, rank=128)):   # down rank above 64
        assert lib.svdq_gemm_w4a4_lora_up_gelu_quant(P(DEV), P(DEV), P(DEV), 64, ctypes.byref(up), ctypes.byref(down),
                                                     P(DEV), P(DEV), P(DEV), P(DEV), 1 << 30, None) == INVALID
    down = _layer(N=256, K=512, rank=32)
    need = lib.svdq_mlp_workspace_bytes(64, 512, 32)
    assert need == 2 * 64 * 32 * 4  # two 256-column tiles of fp32 partials
    assert lib.svdq_gemm_w4a4_lora_up_gelu_quant(P(DEV), P(DEV), P(DEV), 64, ctypes.byref(up), ctypes.byref(down),
                                                 P(DEV), P(DEV), P(DEV), P(DEV), need - 4, None) == INVALID
    assert lib.svdq_gemm_w4a4_lora_up_gelu_quant(P(DEV), P(DEV), P(DEV), 64, ctypes.byref(up), ctypes.byref(down),
                                                 P(DEV), P(DEV), P(DEV), P(DEV), need, None) == UNSUPPORTED
    assert lib.svdq_mlp_workspace_bytes(64, 500, 32) == 0
    assert lib.svdq_mlp_workspace_bytes(64, 512, 128) == 0


def test_awq_gemv_size_limits(lib, unsupported):
    # K up to 12288 (staged activations beside a ring of at least two weight runs), 1..8 tokens
    P = _p
    call = lambda M, K: lib.svdq_awq_gemv_w4a16(P(DEV), M, P(DEV), P(DEV), None, 64, K, P(DEV), None)  # noqa: E731
    assert call(1, 12288) == UNSUPPORTED
    assert call(8, 3072) == UNSUPPORTED
    assert call(1, 12352) == INVALID
    assert call(9, 3072) == INVALID
    assert call(0, 3072) == INVALID


def test_null_layer_is_rejected(lib, unsupported):
    assert lib.svdq_quant_act_lora_down(_p(DEV), 16, None, _p(DEV), _p(DEV), _p(DEV), None) == INVALID
    assert lib.svdq_gemm_w4a4_lora_up(_p(DEV), _p(DEV), _p(DEV), 16, None, _p(DEV), None) == INVALID


def test_misaligned_pointers_are_rejected_before_the_device(lib, unsupported):
    layer = _layer()
    L = ctypes.byref(layer)
    assert lib.svdq_quant_act_lora_down(_p(ODD), 256, L, _p(DEV), _p(DEV), _p(DEV), None) == MISALIGNED
    assert lib.svdq_gemm_w4a4_lora_up(_p(DEV), _p(DEV), _p(DEV), 256, L, _p(ODD), None) == MISALIGNED
    assert lib.svdq_quant_act_lora_down(_p(DEV), 256, ctypes.byref(_layer(wq=ODD)), _p(DEV), _p(DEV), _p(DEV),
                                        None) == MISALIGNED


def test_rank_zero_needs_no_branch_buffers(lib, unsupported):
    # rank 0: lora_act and L1t / L2t may be NULL; the call then gets as far as the device check
    layer = _layer(rank=0)
    assert lib.svdq_quant_act_lora_down(_p(DEV), 256, ctypes.byref(layer), _p(DEV), _p(DEV), None, None) == UNSUPPORTED


@pytest.mark.parametrize("rows,K", [(1, 64), (128, 64), (129, 192), (300, 1024), (513, 3072)])
def test_unswizzle_scales_matches_the_layout_statement(lib, rows, K):
    from bit_rank_compensated_b200 import svdq

    rng = np.random.default_rng(rows + K)
    sc = rng.integers(0, 256, (rows, K // 16)).astype(np.uint8)
    blocked = F.scales_to_blocked(sc, (rows + 127) // 128 * 128)
    got = svdq.unswizzle_scales(blocked, rows, K)
    np.testing.assert_array_equal(got, sc)
    np.testing.assert_array_equal(got, F.blocked_to_scales(blocked, rows, K // 16))


def test_unswizzle_scales_rejects_bad_shapes(lib):
    buf = np.zeros(512, np.uint8)
    out = np.zeros(64, np.uint8)
    vp = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    assert lib.svdq_unswizzle_scales(vp(buf), 4, 48, vp(out)) == INVALID
    assert lib.svdq_unswizzle_scales(vp(buf), 0, 64, vp(out)) == INVALID
    assert lib.svdq_unswizzle_scales(None, 4, 64, vp(out)) == INVALID
    assert lib.svdq_unswizzle_scales(vp(buf), 4, 64, None) == INVALID
    assert lib.svdq_unswizzle_scales(vp(buf), 4, 64, vp(out)) == OK
