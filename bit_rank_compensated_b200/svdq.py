"""Thin ctypes binding of libsvdq (include/svdq.h).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
PyTorch provides device memory (tensors) and the current CUDA stream. There is no CPU
fallback: when libsvdq.so is missing or the GPU is not a B200 the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsvdq.so")

SVDQ_OK = 0
STATUS_NAMES = {
    0: "SVDQ_OK", 1: "SVDQ_ERR_INVALID_ARG", 2: "SVDQ_ERR_UNSUPPORTED_ARCH", 3: "SVDQ_ERR_MISALIGNED",
    4: "SVDQ_ERR_CUDA", 5: "SVDQ_ERR_TIMEOUT", 6: "SVDQ_ERR_INTERNAL", 7: "SVDQ_ERR_UNAVAILABLE",
}
RANKS = (0, 16, 32, 64, 128)
GROUP = 16

# Every symbol include/svdq.h declares.
EXPORTED = (
    "svdq_status_string", "svdq_version", "svdq_weight_scale_bytes", "svdq_act_scale_bytes", "svdq_act_absmax",
    "svdq_prepare_workspace_bytes", "svdq_prepare_weights", "svdq_quantize_rows", "svdq_quant_act_lora_down",
    "svdq_gemm_w4a4_lora_up", "svdq_linear_forward", "svdq_linear_forward_host", "svdq_baseline_lora_down",
    "svdq_baseline_quantize", "svdq_baseline_gemm_w4a4", "svdq_baseline_lora_up", "svdq_last_device_error",
    "svdq_smoothing_factors_noalloc", "svdq_selftest_wait_timeout", "svdq_gemm_w4a4_lora_up_qk_norm_rope",
    "svdq_qk_norm_rope", "svdq_awq_quantize_weights", "svdq_awq_gemv_w4a16", "svdq_awq_pack_weights",
    "svdq_awq_packed_weight_bytes", "svdq_awq_packed_sz_bytes", "svdq_prepare_weights_host",
    "svdq_unswizzle_scales", "svdq_test_override_capability", "svdq_mlp_workspace_bytes",
    "svdq_gemm_w4a4_lora_up_gelu_quant", "svdq_gemm_w4a4_lora_up_gelu", "svdq_mlp_forward",
)


class SvdqError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)} ({msg})")
        self.status = status


class LayerStruct(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int32), ("K", ctypes.c_int32), ("rank", ctypes.c_int32), ("group", ctypes.c_int32),
        ("w_tensor_scale", ctypes.c_float), ("x_tensor_scale", ctypes.c_float),
        ("wq", ctypes.c_void_p), ("ws", ctypes.c_void_p), ("inv_lambda", ctypes.c_void_p),
        ("lambda_", ctypes.c_void_p), ("L1t", ctypes.c_void_p), ("L2t", ctypes.c_void_p),
        ("bias", ctypes.c_void_p),
    ]


_lib = None


def load() -> ctypes.CDLL:
    """Loads libsvdq.so (built in-tree by bit_rank_compensated_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with `python -m bit_rank_compensated_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    LP = ctypes.POINTER(LayerStruct)
    sig = {
        "svdq_status_string": ([I], ctypes.c_char_p),
        "svdq_version": ([], I),
        "svdq_weight_scale_bytes": ([I, I], S),
        "svdq_act_scale_bytes": ([I, I], S),
        "svdq_act_absmax": ([P, I, I, P, P], I),
        "svdq_prepare_workspace_bytes": ([I, I, I, ctypes.POINTER(I)], S),
        "svdq_prepare_weights": ([P, P, P, I, I, I, LP, P, S, P], I),
        "svdq_quantize_rows": ([P, I, I, F, I, P, P, P], I),
        "svdq_quant_act_lora_down": ([P, I, LP, P, P, P, P], I),
        "svdq_gemm_w4a4_lora_up": ([P, P, P, I, LP, P, P], I),
        "svdq_linear_forward": ([P, I, LP, P, P, P, P, P], I),
        "svdq_linear_forward_host": ([P, I, LP, P, P, P, P, P, P, P], I),
        "svdq_baseline_lora_down": ([P, I, LP, P, P], I),
        "svdq_baseline_quantize": ([P, I, LP, P, P, P], I),
        "svdq_baseline_gemm_w4a4": ([P, P, I, LP, P, P], I),
        "svdq_baseline_lora_up": ([P, I, LP, P, P], I),
        "svdq_last_device_error": ([P, ctypes.POINTER(ctypes.c_uint32)], I),
        "svdq_selftest_wait_timeout": ([ctypes.c_uint32, P], I),
        "svdq_smoothing_factors_noalloc": ([P, P, I, I, P, P, P, P], I),
        "svdq_gemm_w4a4_lora_up_qk_norm_rope": ([P, P, P, I, LP, I, I, P, P, P, F, P, P], I),
        "svdq_qk_norm_rope": ([P, I, I, I, P, P, P, F, P], I),
        "svdq_awq_quantize_weights": ([P, I, I, P, P, P, P], I),
        "svdq_awq_gemv_w4a16": ([P, I, P, P, P, I, I, P, P], I),
        "svdq_awq_pack_weights": ([P, P, P, I, I, P, P, P], I),
        "svdq_awq_packed_weight_bytes": ([I, I], S),
        "svdq_awq_packed_sz_bytes": ([I, I], S),
        "svdq_prepare_weights_host": ([P, P, P, I, I, I, LP, P, P], I),
        "svdq_unswizzle_scales": ([P, I, I, P], I),
        "svdq_test_override_capability": ([I, I], I),
        "svdq_mlp_workspace_bytes": ([I, I, I], S),
        "svdq_gemm_w4a4_lora_up_gelu_quant": ([P, P, P, I, LP, LP, P, P, P, P, S, P], I),
        "svdq_gemm_w4a4_lora_up_gelu": ([P, P, P, I, LP, P, P], I),
        "svdq_mlp_forward": ([P, I, LP, LP, P, P, P, P, P, P, P, S, P, P], I),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def _check(fn: str, status: int):
    if status != SVDQ_OK:
        raise SvdqError(fn, status, load().svdq_status_string(status).decode())


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def weight_scale_bytes(N: int, K: int) -> int:
    return load().svdq_weight_scale_bytes(N, K)


def act_scale_bytes(M: int, K: int) -> int:
    return load().svdq_act_scale_bytes(M, K)


class Layer:
    """Device buffers of one prepared layer (tensors) plus the C struct that points at them."""

    def __init__(self, N: int, K: int, rank: int, device="cuda", with_bias: bool = True):
        if rank not in RANKS:
            raise ValueError(f"rank must be one of {RANKS}")
        self.N, self.K, self.rank = N, K, rank
        u8 = dict(dtype=torch.uint8, device=device)
        self.wq = torch.empty(N * K // 2, **u8)
        self.ws = torch.empty(weight_scale_bytes(N, K), **u8)
        self.inv_lambda = torch.empty(K, dtype=torch.float32, device=device)
        self.lam = torch.empty(K, dtype=torch.float32, device=device)
        self.L1t = torch.empty(max(rank, 1) * K, dtype=torch.bfloat16, device=device) if rank else None
        self.L2t = torch.empty(N * max(rank, 1), dtype=torch.bfloat16, device=device) if rank else None
        self.bias = torch.zeros(N, dtype=torch.float32, device=device) if with_bias else None
        self.s = LayerStruct()
        self.s.N, self.s.K, self.s.rank, self.s.group = N, K, rank, GROUP
        self.s.w_tensor_scale = 1.0
        self.s.x_tensor_scale = 1.0
        self._sync_ptrs()

    def _sync_ptrs(self):
        self.s.wq = self.wq.data_ptr()
        self.s.ws = self.ws.data_ptr()
        self.s.inv_lambda = self.inv_lambda.data_ptr()
        self.s.lambda_ = self.lam.data_ptr()
        self.s.L1t = self.L1t.data_ptr() if self.L1t is not None else None
        self.s.L2t = self.L2t.data_ptr() if self.L2t is not None else None
        self.s.bias = self.bias.data_ptr() if self.bias is not None else None

    @property
    def s_w(self) -> float:
        return float(self.s.w_tensor_scale)

    @property
    def s_x(self) -> float:
        return float(self.s.x_tensor_scale)

    @classmethod
    def from_arrays(cls, *, N, K, rank, wq, ws, inv_lambda, L1t, L2t, bias, s_w, s_x, lam=None, device="cuda"):
        """Builds a layer from already prepared host arrays (numpy): packed codes, block-layout
        scales, inv_lambda, L1t / L2t as bf16 bit patterns (uint16), bias (or None)."""
        import numpy as np

        L = cls(N, K, rank, device=device, with_bias=bias is not None)
        L.wq.copy_(torch.from_numpy(np.ascontiguousarray(wq, dtype=np.uint8).reshape(-1)))
        L.ws.copy_(torch.from_numpy(np.ascontiguousarray(ws, dtype=np.uint8).reshape(-1)))
        L.inv_lambda.copy_(torch.from_numpy(np.ascontiguousarray(inv_lambda, dtype=np.float32)))
        if lam is not None:
            L.lam.copy_(torch.from_numpy(np.ascontiguousarray(lam, dtype=np.float32)))
        if rank:
            L.L1t.view(torch.int16).copy_(torch.from_numpy(np.ascontiguousarray(L1t, dtype=np.uint16).reshape(-1).view(np.int16)))
            L.L2t.view(torch.int16).copy_(torch.from_numpy(np.ascontiguousarray(L2t, dtype=np.uint16).reshape(-1).view(np.int16)))
        if bias is not None:
            L.bias.copy_(torch.from_numpy(np.ascontiguousarray(bias, dtype=np.float32)))
        L.s.w_tensor_scale = float(s_w)
        L.s.x_tensor_scale = float(s_x)
        return L


def act_absmax(X: torch.Tensor, stream=None) -> torch.Tensor:
    M, K = X.shape
    out = torch.empty(K, dtype=torch.float32, device=X.device)
    _check("svdq_act_absmax", load().svdq_act_absmax(_ptr(X), M, K, _ptr(out), _stream(stream)))
    return out


def prepare_workspace_bytes(N: int, K: int, rank: int) -> int:
    st = ctypes.c_int(0)
    n = load().svdq_prepare_workspace_bytes(N, K, rank, ctypes.byref(st))
    _check("svdq_prepare_workspace_bytes", st.value)
    return n


def prepare_weights(W: torch.Tensor, bias: torch.Tensor | None, act_absmax_: torch.Tensor, rank: int,
                    stream=None) -> Layer:
    N, K = W.shape
    L = Layer(N, K, rank, device=W.device, with_bias=bias is not None)
    ws = torch.empty(prepare_workspace_bytes(N, K, rank), dtype=torch.uint8, device=W.device)
    _check("svdq_prepare_weights", load().svdq_prepare_weights(
        _ptr(W), _ptr(bias), _ptr(act_absmax_), N, K, rank, ctypes.byref(L.s), _ptr(ws), ws.numel(),
        _stream(stream)))
    del ws
    return L


def prepare_weights_host(W, bias, act_absmax_, rank: int, return_residual: bool = False, device="cuda",
                         stream=None):
    """svdq_prepare_weights_host: prepare a layer from host (numpy) arrays. With
    return_residual the fp32 residual R (N x K numpy array) the weight quantizer read comes back too."""
    import numpy as np

    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    ax = np.ascontiguousarray(act_absmax_, dtype=np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    L = Layer(N, K, rank, device=device, with_bias=b is not None)
    R = np.empty((N, K), dtype=np.float32) if return_residual else None
    _check("svdq_prepare_weights_host", load().svdq_prepare_weights_host(
        W.ctypes.data_as(ctypes.c_void_p), None if b is None else b.ctypes.data_as(ctypes.c_void_p),
        ax.ctypes.data_as(ctypes.c_void_p), N, K, rank, ctypes.byref(L.s),
        None if R is None else R.ctypes.data_as(ctypes.c_void_p), _stream(stream)))
    return (L, R) if return_residual else L


def unswizzle_scales(blocked, rows: int, K: int):
    """svdq_unswizzle_scales: group scales of `rows` rows from the block layout (host bytes, e.g. a
    buffer copied back from the device) to a row-major numpy array rows x K/16."""
    import numpy as np

    buf = np.ascontiguousarray(np.asarray(blocked, dtype=np.uint8).reshape(-1))
    need = (rows + 127) // 128 * 128 * (K // 16)
    if buf.size < need:
        raise ValueError(f"blocked scale buffer holds {buf.size} bytes, {need} needed")
    out = np.empty((rows, K // 16), dtype=np.uint8)
    _check("svdq_unswizzle_scales", load().svdq_unswizzle_scales(
        buf.ctypes.data_as(ctypes.c_void_p), rows, K, out.ctypes.data_as(ctypes.c_void_p)))
    return out


def test_override_capability(major: int, minor: int = 0) -> None:
    """Test hook: make the library treat the GPU as compute capability major.minor (major < 0
    removes the override)."""
    _check("svdq_test_override_capability", load().svdq_test_override_capability(int(major), int(minor)))


def smoothing_factors_noalloc(W: torch.Tensor, act_absmax_: torch.Tensor, lam=None, inv_lam=None, s_x=None,
                              stream=None):
    """lambda, inv_lambda and the activation tensor scale of a layer, computed without any
    device allocation inside the library (its scratch is a static device array, K <= 65536).
    Output tensors may be passed in (the call then allocates nothing at all)."""
    N, K = W.shape
    lam = torch.empty(K, dtype=torch.float32, device=W.device) if lam is None else lam
    inv_lam = torch.empty(K, dtype=torch.float32, device=W.device) if inv_lam is None else inv_lam
    s_x = torch.empty(1, dtype=torch.float32, device=W.device) if s_x is None else s_x
    _check("svdq_smoothing_factors_noalloc", load().svdq_smoothing_factors_noalloc(
        _ptr(W), _ptr(act_absmax_), N, K, _ptr(lam), _ptr(inv_lam), _ptr(s_x), _stream(stream)))
    return lam, inv_lam, s_x


def quantize_rows(A: torch.Tensor, s: float, row_pad: int = 256, stream=None):
    rows, K = A.shape
    codes = torch.empty(rows * K // 2, dtype=torch.uint8, device=A.device)
    pad = (rows + row_pad - 1) // row_pad * row_pad
    scales = torch.empty(pad * K // 16, dtype=torch.uint8, device=A.device)
    _check("svdq_quantize_rows", load().svdq_quantize_rows(
        _ptr(A), rows, K, float(s), row_pad, _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def alloc_activations(M: int, layer: Layer, device="cuda"):
    xq = torch.empty(M * layer.K // 2, dtype=torch.uint8, device=device)
    xs = torch.empty(act_scale_bytes(M, layer.K), dtype=torch.uint8, device=device)
    # lora_act rows hold [hi | lo] bf16 planes of the pre-scaled down-projection
    la = torch.empty(M * 2 * layer.rank, dtype=torch.bfloat16, device=device) if layer.rank else None
    return xq, xs, la


def quant_act_lora_down(X: torch.Tensor, layer: Layer, xq=None, xs=None, lora_act=None, stream=None):
    M = X.shape[0]
    if xq is None:
        xq, xs, lora_act = alloc_activations(M, layer, X.device)
    _check("svdq_quant_act_lora_down", load().svdq_quant_act_lora_down(
        _ptr(X), M, ctypes.byref(layer.s), _ptr(xq), _ptr(xs), _ptr(lora_act), _stream(stream)))
    return xq, xs, lora_act


def gemm_w4a4_lora_up(xq, xs, lora_act, M: int, layer: Layer, Y=None, stream=None):
    if Y is None:
        Y = torch.empty(M, layer.N, dtype=torch.bfloat16, device=xq.device)
    _check("svdq_gemm_w4a4_lora_up", load().svdq_gemm_w4a4_lora_up(
        _ptr(xq), _ptr(xs), _ptr(lora_act), M, ctypes.byref(layer.s), _ptr(Y), _stream(stream)))
    return Y


def gemm_w4a4_lora_up_qk_norm_rope(xq, xs, lora_act, M: int, layer: Layer, heads: int, norm_q, norm_k, rope,
                                   eps: float = 1e-6, Y=None, stream=None, head_dim: int = 128):
    """K2 with the fused QKV output stage: Y = [Q | K | V], Q and K heads RMS-normalized with
    norm_q / norm_k (fp32 [head_dim]) and turned by the (cos, sin) table rope (fp32 [M, 64, 2])."""
    if Y is None:
        Y = torch.empty(M, layer.N, dtype=torch.bfloat16, device=xq.device)
    _check("svdq_gemm_w4a4_lora_up_qk_norm_rope", load().svdq_gemm_w4a4_lora_up_qk_norm_rope(
        _ptr(xq), _ptr(xs), _ptr(lora_act), M, ctypes.byref(layer.s), heads, head_dim, _ptr(norm_q), _ptr(norm_k),
        _ptr(rope), float(eps), _ptr(Y), _stream(stream)))
    return Y


def qk_norm_rope(Y, heads: int, norm_q, norm_k, rope, eps: float = 1e-6, stream=None, head_dim: int = 128):
    """Unfused step: normalizes and rotates the Q and K sections of a bf16 Y in place."""
    _check("svdq_qk_norm_rope", load().svdq_qk_norm_rope(
        _ptr(Y), Y.shape[0], heads, head_dim, _ptr(norm_q), _ptr(norm_k), _ptr(rope), float(eps), _stream(stream)))
    return Y


def awq_quantize_weights(W: torch.Tensor, stream=None):
    """int4 codes (N x K/2 uint8), fp16 scales (N x K/64), zero points (N x K/64 uint8) of W (fp32)."""
    N, K = W.shape
    wq = torch.empty(N, K // 2, dtype=torch.uint8, device=W.device)
    scales = torch.empty(N, K // 64, dtype=torch.float16, device=W.device)
    zeros = torch.empty(N, K // 64, dtype=torch.uint8, device=W.device)
    _check("svdq_awq_quantize_weights", load().svdq_awq_quantize_weights(
        _ptr(W), N, K, _ptr(wq), _ptr(scales), _ptr(zeros), _stream(stream)))
    return wq, scales, zeros


def awq_pack_weights(wq, scales, zeros, stream=None):
    """The GEMV's tile layout of quantized weights: (wq_packed, sz_packed) uint8 device buffers."""
    N, K = wq.shape[0], 2 * wq.shape[1]
    lib = load()
    wt = torch.empty(lib.svdq_awq_packed_weight_bytes(N, K), dtype=torch.uint8, device=wq.device)
    szt = torch.empty(lib.svdq_awq_packed_sz_bytes(N, K), dtype=torch.uint8, device=wq.device)
    _check("svdq_awq_pack_weights", lib.svdq_awq_pack_weights(
        _ptr(wq), _ptr(scales), _ptr(zeros), N, K, _ptr(wt), _ptr(szt), _stream(stream)))
    return wt, szt


class AwqLinear:
    """A packed awq_w4a16 weight (N x K) with its bias, ready for awq_gemv_w4a16. Built at load
    time: the constructor waits for the packing to finish, since the GEMV may read the packed
    weights before the kernel just before it on its stream has finished."""

    def __init__(self, wq, scales, zeros, bias=None, stream=None):
        self.N, self.K = wq.shape[0], 2 * wq.shape[1]
        self.wt, self.szt = awq_pack_weights(wq, scales, zeros, stream)
        self.bias = bias
        (stream if stream is not None else torch.cuda.current_stream(wq.device)).synchronize()

    @classmethod
    def from_float(cls, W: torch.Tensor, bias=None, stream=None):
        return cls(*awq_quantize_weights(W, stream), bias=bias, stream=stream)


def awq_gemv_w4a16(X: torch.Tensor, lin: "AwqLinear", Y=None, stream=None):
    """Y = bf16(X W_hat^T + bias) for a bf16 X of 1..8 rows."""
    M, K = X.shape
    if Y is None:
        Y = torch.empty(M, lin.N, dtype=torch.bfloat16, device=X.device)
    _check("svdq_awq_gemv_w4a16", load().svdq_awq_gemv_w4a16(
        _ptr(X), M, _ptr(lin.wt), _ptr(lin.szt), _ptr(lin.bias), lin.N, K, _ptr(Y), _stream(stream)))
    return Y


def mlp_workspace_bytes(M: int, up: Layer, down: Layer) -> int:
    return load().svdq_mlp_workspace_bytes(M, up.N, down.rank)


def alloc_mlp_workspace(M: int, up: Layer, down: Layer, device="cuda"):
    n = mlp_workspace_bytes(M, up, down)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def gemm_w4a4_lora_up_gelu_quant(xq, xs, lora_act, M: int, up: Layer, down: Layer, bufs_down=None, workspace=None,
                                 stream=None):
    """The fused MLP pair's middle: the down layer's (xq, xs, lora_act) from GELU(up layer output)."""
    if bufs_down is None:
        bufs_down = alloc_activations(M, down, xq.device)
    if workspace is None:
        workspace = alloc_mlp_workspace(M, up, down, xq.device)
    xq_d, xs_d, la_d = bufs_down
    _check("svdq_gemm_w4a4_lora_up_gelu_quant", load().svdq_gemm_w4a4_lora_up_gelu_quant(
        _ptr(xq), _ptr(xs), _ptr(lora_act), M, ctypes.byref(up.s), ctypes.byref(down.s), _ptr(xq_d), _ptr(xs_d),
        _ptr(la_d), _ptr(workspace), workspace.numel(), _stream(stream)))
    return bufs_down


def gemm_w4a4_lora_up_gelu(xq, xs, lora_act, M: int, layer: Layer, H=None, stream=None):
    """H = bf16(GELU(layer output)): the unfused pair's first layer."""
    if H is None:
        H = torch.empty(M, layer.N, dtype=torch.bfloat16, device=xq.device)
    _check("svdq_gemm_w4a4_lora_up_gelu", load().svdq_gemm_w4a4_lora_up_gelu(
        _ptr(xq), _ptr(xs), _ptr(lora_act), M, ctypes.byref(layer.s), _ptr(H), _stream(stream)))
    return H


def mlp_forward(X, up: Layer, down: Layer, bufs=None, bufs_down=None, workspace=None, Z=None, stream=None):
    """The fused FLUX feed-forward pair Z = down(GELU(up(X)))."""
    M = X.shape[0]
    xq, xs, la = bufs if bufs is not None else alloc_activations(M, up, X.device)
    xq_d, xs_d, la_d = bufs_down if bufs_down is not None else alloc_activations(M, down, X.device)
    if workspace is None:
        workspace = alloc_mlp_workspace(M, up, down, X.device)
    if Z is None:
        Z = torch.empty(M, down.N, dtype=torch.bfloat16, device=X.device)
    _check("svdq_mlp_forward", load().svdq_mlp_forward(
        _ptr(X), M, ctypes.byref(up.s), ctypes.byref(down.s), _ptr(xq), _ptr(xs), _ptr(la), _ptr(xq_d), _ptr(xs_d),
        _ptr(la_d), _ptr(workspace), workspace.numel(), _ptr(Z), _stream(stream)))
    return Z


def linear_forward(X: torch.Tensor, layer: Layer, bufs=None, Y=None, stream=None):
    M = X.shape[0]
    xq, xs, la = bufs if bufs is not None else alloc_activations(M, layer, X.device)
    if Y is None:
        Y = torch.empty(M, layer.N, dtype=torch.bfloat16, device=X.device)
    _check("svdq_linear_forward", load().svdq_linear_forward(
        _ptr(X), M, ctypes.byref(layer.s), _ptr(xq), _ptr(xs), _ptr(la), _ptr(Y), _stream(stream)))
    return Y


def linear_forward_host(X_host: torch.Tensor, layer: Layer, X_dev, bufs, Y_dev, Y_host, stream=None):
    M = X_host.shape[0]
    xq, xs, la = bufs
    _check("svdq_linear_forward_host", load().svdq_linear_forward_host(
        _ptr(X_host), M, ctypes.byref(layer.s), _ptr(X_dev), _ptr(xq), _ptr(xs), _ptr(la), _ptr(Y_dev),
        _ptr(Y_host), _stream(stream)))
    return Y_host


def baseline_lora_down(X, layer, lora_act, stream=None):
    _check("svdq_baseline_lora_down", load().svdq_baseline_lora_down(
        _ptr(X), X.shape[0], ctypes.byref(layer.s), _ptr(lora_act), _stream(stream)))


def baseline_quantize(X, layer, xq, xs, stream=None):
    _check("svdq_baseline_quantize", load().svdq_baseline_quantize(
        _ptr(X), X.shape[0], ctypes.byref(layer.s), _ptr(xq), _ptr(xs), _stream(stream)))


def baseline_gemm_w4a4(xq, xs, M, layer, Y, stream=None):
    _check("svdq_baseline_gemm_w4a4", load().svdq_baseline_gemm_w4a4(
        _ptr(xq), _ptr(xs), M, ctypes.byref(layer.s), _ptr(Y), _stream(stream)))


def baseline_lora_up(lora_act, M, layer, Y, stream=None):
    _check("svdq_baseline_lora_up", load().svdq_baseline_lora_up(
        _ptr(lora_act), M, ctypes.byref(layer.s), _ptr(Y), _stream(stream)))


def unfused_forward(X, layer, bufs, Y, stream=None):
    """The naive branch of the unfused baseline: four separate kernels."""
    xq, xs, la = bufs
    M = X.shape[0]
    if layer.rank:
        baseline_lora_down(X, layer, la, stream)
    baseline_quantize(X, layer, xq, xs, stream)
    baseline_gemm_w4a4(xq, xs, M, layer, Y, stream)
    if layer.rank:
        baseline_lora_up(la, M, layer, Y, stream)
    return Y


def selftest_wait_timeout(limit_us: int, stream=None) -> None:
    """Runs the failure-path self-test kernel (bounded waits on an mbarrier nothing signals);
    read the recorded timeout with last_device_error()."""
    _check("svdq_selftest_wait_timeout", load().svdq_selftest_wait_timeout(int(limit_us), _stream(stream)))


def last_device_error(stream=None) -> int:
    code = ctypes.c_uint32(0)
    st = load().svdq_last_device_error(_stream(stream), ctypes.byref(code))
    if st not in (SVDQ_OK, 5):
        _check("svdq_last_device_error", st)
    return int(code.value)
