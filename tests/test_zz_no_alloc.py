"""svdq_smoothing_factors_noalloc: the smoothing stage for callers that cannot allocate device
memory (a fixed memory budget, or a framework that forbids allocations after start-up).

The entry point keeps its scratch in a static device array inside the library. This test calls
it through the C ABI with preallocated outputs, twice in a row on different inputs (the second
call must not see the first call's scratch), and compares lambda, inv_lambda and the activation
tensor scale with what svdq_prepare_weights computes for the same inputs (bit for bit, the
tolerance our tests use for these quantities). It lives in its own file, collected last.
"""
import ctypes

import numpy as np
import pytest

from synth import LayerShape, make_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _inputs(seed, scale):
    Xb, W, b, _ = make_inputs(LayerShape("noalloc", 192, 1024, 320, 0, "spiky4"), seed=seed)
    Xd = torch.from_numpy(Xb.view(np.int16)).cuda().view(torch.bfloat16)
    return Xd, torch.from_numpy(W * scale).cuda(), torch.from_numpy(b).cuda()


def _noalloc(lib, W, ax, lam, inv_lam, s_x):
    N, K = W.shape
    st = lib.load().svdq_smoothing_factors_noalloc(
        ctypes.c_void_p(W.data_ptr()), ctypes.c_void_p(ax.data_ptr()), N, K, ctypes.c_void_p(lam.data_ptr()),
        ctypes.c_void_p(inv_lam.data_ptr()), ctypes.c_void_p(s_x.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return st


def test_noalloc_smoothing_matches_prepare_twice():
    from bit_rank_compensated_b200 import svdq as lib

    assert torch.cuda.is_available()
    K = 1024
    lam = torch.empty(K, dtype=torch.float32, device="cuda")
    inv_lam = torch.empty(K, dtype=torch.float32, device="cuda")
    s_x = torch.empty(1, dtype=torch.float32, device="cuda")
    # second call: smaller activation maxima, so a stale running maximum would show up
    for seed, scale, xscale in [(0, 4.0, 1.0), (1, 0.25, 0.01)]:
        Xd, W, b = _inputs(seed, scale)
        ax = lib.act_absmax(Xd) * xscale
        assert _noalloc(lib, W, ax, lam, inv_lam, s_x) == 0
        ref = lib.prepare_weights(W, b, ax, 0)
        torch.cuda.synchronize()
        assert torch.equal(lam, ref.lam)
        assert torch.equal(inv_lam, ref.inv_lambda)
        assert float(s_x.item()) == ref.s_x
    assert lib.last_device_error() == 0


def test_noalloc_rejects_oversized_k():
    from bit_rank_compensated_b200 import svdq as lib

    K = 65536 + 64
    W = torch.zeros(16, K, dtype=torch.float32, device="cuda")
    ax = torch.ones(K, dtype=torch.float32, device="cuda")
    out = torch.empty(K, dtype=torch.float32, device="cuda")
    s_x = torch.empty(1, dtype=torch.float32, device="cuda")
    assert _noalloc(lib, W, ax, out, out, s_x) == 1  # SVDQ_ERR_INVALID_ARG, nothing launched
