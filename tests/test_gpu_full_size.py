"""Parity at the full sizes the benchmark reports, in the launch configuration it times.

Workloads (FLUX-like linear layers at rank 32): the fused QKV projection (4608 tokens, 3072 ->
9216), the MLP up-projection (3072 -> 12288), the MLP down-projection (12288 -> 3072) and the
largest token count of the sweep (16384 tokens, 3072 -> 3072). These take the activation
kernel's multi-CTA cluster splits along K (up to 192 chunks of 64 columns), the GEMM's 48 4-bit
steps per tile and grids of more than one wave, which the small parity cases do not reach.

Per workload, with the oracle's own prepared layer on the device:
  * every row's NVFP4 codes and e4m3 group scales from svdq_quant_act_lora_down, bit for bit
    (the padding rows' scales zero), and the down-projection of every row within 1e-3;
  * the layer output for at least 512 rows spread over every 64-row activation tile, every row
    position inside a tile (so every owner of the split-K reduction) and the whole last 256-row
    GEMM tile, within the output tolerance max |Y - Y_ref| / max(|Y_ref|, 1e-2 rms) <= 1e-2.
And the library's own prepare at full size (svdq_prepare_weights_host): smoothing factors and
tensor scales bit for bit, the bf16 branch factors bit for bit up to the two SVD routes' rare
last-bit differences, the residual close to the oracle's, and the weight codes bit for bit
wherever the two residuals agree; the weight quantizer itself on the oracle's residual at full
size, bit for bit.
"""
import numpy as np
import pytest

from oracle import svdq_oracle as O
from synth import CONFIGS, bf16_bits_to_f32, make_inputs
from tests.gpu_helpers import (Y_TOL, alpha32, bf16_tensor_to_np, fro_rel, lora_pair_value, oracle_layer_arrays,
                               rel_err_floor, to_device_layer, x_to_device)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

FULL = ["qkv", "mlp_up", "mlp_down", "sweep_m16384"]


@pytest.fixture(scope="module")
def lib():
    from bit_rank_compensated_b200 import svdq

    svdq.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return svdq


@pytest.fixture(scope="module", params=FULL)
def case(request):
    shape = CONFIGS[request.param]
    Xb, W, b, _ = make_inputs(shape, seed=0)
    X = bf16_bits_to_f32(Xb).astype(np.float64)
    layer_o = O.prepare(W, b, O.calibration_absmax(X), shape.rank)
    codes, scales, La = O.quant_act_lora_down(X, layer_o)
    yield dict(shape=shape, Xb=Xb, X=X, W=W, b=b, layer=layer_o, codes=codes, scales=scales, La=La)
    torch.cuda.empty_cache()


def sample_rows(M: int) -> np.ndarray:
    """Rows spread over every 64-row activation tile: eight per tile, one in each 8-row group at
    an offset that cycles with the tile (so every row position 0..63 occurs), plus every row of
    the last 256-row GEMM tile."""
    rows = set()
    for t in range((M + 63) // 64):
        o = t % 8
        for i in range(8):
            m = t * 64 + o + 8 * i
            if m < M:
                rows.add(m)
    rows.update(range((M - 1) // 256 * 256, M))
    return np.array(sorted(rows))


def test_sample_covers_tiles_and_positions():
    for M in (4608, 16384, 300):
        r = sample_rows(M)
        assert set(np.unique(r // 64)) == set(range((M + 63) // 64))
        assert M < 512 or set(np.unique(r % 64)) == set(range(64))
        assert M < 512 or len(r) >= 512
        assert r.max() == M - 1


def test_full_size_activations_and_output(lib, case):
    shape, X, layer_o = case["shape"], case["X"], case["layer"]
    M, K, N, r = shape.M, shape.K, shape.N, shape.rank
    Ld = to_device_layer(layer_o)
    Xd = x_to_device(case["Xb"])
    xq, xs, la = lib.alloc_activations(M, Ld)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    # the two calls the benchmark times, on the current stream
    lib.quant_act_lora_down(Xd, Ld, xq, xs, la)
    lib.gemm_w4a4_lora_up(xq, xs, la, M, Ld, Y)
    torch.cuda.synchronize()
    assert lib.last_device_error() == 0

    # every row: codes and scales bit for bit, padding scales zero
    np.testing.assert_array_equal(xq.cpu().numpy().reshape(M, K // 2), O.pack_codes(case["codes"]))
    Mp = (M + 127) // 128 * 128
    sc = lib.unswizzle_scales(xs.cpu().numpy(), Mp, K)
    np.testing.assert_array_equal(sc[:M], case["scales"])
    assert not sc[M:].any()
    # every row: the pre-scaled down-projection (hi + lo) within 1e-3 of the fp64 value
    got_la = lora_pair_value(la, M, r)
    assert rel_err_floor(got_la, case["La"] / alpha32(layer_o)) <= 1e-3

    rows = sample_rows(M)
    Y_ref = O.gemm_w4a4_lora_up(case["codes"][rows], case["scales"][rows], case["La"][rows], layer_o)
    got = bf16_tensor_to_np(Y[torch.from_numpy(rows).cuda()])
    err = rel_err_floor(got, Y_ref)
    assert err <= Y_TOL, f"{shape.name}: max floor-relative error {err:.3e} over {len(rows)} rows"
    assert fro_rel(got, Y_ref) <= 5e-3


def test_full_size_weight_quantizer(lib, case):
    # svdq_quantize_rows on the oracle's fp32 residual at full size: codes and scales bit for bit
    layer_o = case["layer"]
    R = torch.from_numpy(np.ascontiguousarray(layer_o.R.astype(np.float32))).cuda()
    codes, scales = lib.quantize_rows(R, layer_o.s_w, 256)
    torch.cuda.synchronize()
    N, K = layer_o.N, layer_o.K
    np.testing.assert_array_equal(codes.cpu().numpy().reshape(N, K // 2), O.pack_codes(layer_o.w_codes))
    np.testing.assert_array_equal(lib.unswizzle_scales(scales.cpu().numpy(), N, K), layer_o.w_scales)


def test_full_size_library_prepare(lib, case):
    shape, layer_o = case["shape"], case["layer"]
    N, K, r = shape.N, shape.K, shape.rank
    ax = lib.act_absmax(x_to_device(case["Xb"])).cpu().numpy()
    np.testing.assert_array_equal(ax, O.calibration_absmax(case["X"]).astype(np.float32))
    L, R = lib.prepare_weights_host(case["W"], case["b"], ax, r, return_residual=True)
    np.testing.assert_array_equal(L.lam.cpu().numpy(), layer_o.lam.astype(np.float32))
    np.testing.assert_array_equal(L.inv_lambda.cpu().numpy(), layer_o.inv_lam.astype(np.float32))
    assert L.s_x == np.float32(layer_o.s_x)
    ref = oracle_layer_arrays(layer_o)
    # two fp64 SVD routes (eigen-decomposition of the Gram matrix, LAPACK's SVD) agree to ~1e-13
    # relative, far below a bf16 step: the rounded factors may differ only where a value sits
    # within that distance of a rounding boundary
    l1 = L.L1t.view(torch.int16).cpu().numpy().view(np.uint16).reshape(r, K)
    l2 = L.L2t.view(torch.int16).cpu().numpy().view(np.uint16).reshape(N, r)
    assert np.mean(l1 != ref["L1t"]) <= 1e-3 and np.mean(l2 != ref["L2t"]) <= 1e-3
    R_o = layer_o.R.astype(np.float32)
    assert fro_rel(R, R_o) <= 1e-3
    # weight codes where the two residuals agree on the whole group (and the tensor scales agree)
    assert L.s_w == np.float32(layer_o.s_w)
    same = np.all((R == R_o).reshape(N, K // 16, 16), axis=2)
    assert same.mean() >= 0.95
    wq = O.unpack_codes(L.wq.cpu().numpy().reshape(N, K // 2)).reshape(N, K // 16, 16)
    np.testing.assert_array_equal(wq[same], layer_o.w_codes.reshape(N, K // 16, 16)[same])
    ws = lib.unswizzle_scales(L.ws.cpu().numpy(), N, K)
    np.testing.assert_array_equal(ws[same], layer_o.w_scales[same])
