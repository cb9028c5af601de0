"""Exhaustive sweep of the activation quantizer's input domain through the activation kernel.

"Nunchaku Lite in Diffusers", native loading, quantization_config (nvfp4, group_size 16): the
activation codes and scales are integers decided by floating point, so they must equal the
oracle's bit for bit for every input, not only for typical ones. The kernel's input is a bf16 X
times an fp32 inv_lambda, so every finite bf16 value (65 280 bit patterns: both signs, zero,
subnormals, every normal binade up to the largest finite value) is put through
svdq_quant_act_lora_down:
  * in several groups each: next to an anchor of |v| F (F from 1 to 17, rounded up to bf16, so
    that v / (group scale) lands anywhere in the e2m1 range, on and around its rounding
    thresholds) and to v's fourteen nearest bf16 neighbours;
  * multiplied by several inv_lambda values (powers of two and values like fp32(1/3), fp32(0.1)
    and 1 - 2^-24 whose products round);
  * under tensor scales s_x that walk the whole supported range [2^-116, 2^116] in windows of
    2^16, exact powers of two and inexact ones (1.37 x 2^e) alternating, each window holding the
    values whose magnitude lies within 2^16 of it (the rest only saturate or quantize to zero,
    which the widest run below covers).
The codes and padded block scales are compared with oracle.nvfp4_quantize(fp32(X inv_lambda), s_x)
bit for bit.
"""
import numpy as np
import pytest

from oracle import svdq_oracle as O
from synth import bf16_bits_to_f32, f32_to_bf16_bits
from tests.gpu_helpers import x_to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

K = 1024
GROUPS_PER_ROW = K // 16
ANCHOR_FACTORS = (1.0, 1.5, 2.75, 5.0, 9.0, 17.0)
# inverse smoothing factors: all <= 1, so |X inv_lambda| stays finite for every bf16 X
INV_LAMBDAS = np.array([1.0, 0.5, 0.75, 1.0 / 3.0, 1.0 / 7.0, 1.0 - 2.0 ** -24, 0.1, 2.0 ** -7 * 1.1],
                       dtype=np.float32)


def finite_bf16_bits():
    b = np.arange(65536, dtype=np.uint32)
    return b[((b >> 7) & 0xFF) != 0xFF].astype(np.uint16)


def _bf16_round_up(mag):
    """Smallest bf16 value >= mag (mag >= 0 fp64), saturating at the largest finite bf16."""
    b = f32_to_bf16_bits(np.minimum(mag, 3.3895313892515355e38).astype(np.float32))
    v = bf16_bits_to_f32(b).astype(np.float64)
    b = np.where(v < mag, b + 1, b).astype(np.uint16)
    b = np.where(((b >> 7) & 0xFF) == 0xFF, np.uint16(0x7F7F), b)
    return b


def sweep_groups(vbits, rng):
    """Groups (rows of 16 bf16 bit patterns): per value v and anchor factor F, [anchor, v, 14
    neighbours of v], signs of anchor and neighbours random."""
    n = vbits.size
    out = []
    mag = np.abs(bf16_bits_to_f32(vbits).astype(np.float64))
    for F in ANCHOR_FACTORS:
        g = np.empty((n, 16), dtype=np.uint16)
        anchor_mag = np.where(mag > 0, mag * F, F)
        g[:, 0] = _bf16_round_up(anchor_mag) | (rng.integers(0, 2, n).astype(np.uint16) << 15)
        g[:, 1] = vbits
        mbits = vbits & 0x7FFF
        for i, d in enumerate([1, -1, 2, -2, 3, -3, 4, -4, 5, -5, 6, -6, 7, -7]):
            nb = mbits.astype(np.int32) + d
            nb = np.where((nb < 0) | (((nb >> 7) & 0xFF) == 0xFF), mbits, nb).astype(np.uint16)
            g[:, 2 + i] = nb | (rng.integers(0, 2, n).astype(np.uint16) << 15)
        out.append(g)
    return np.concatenate(out, axis=0)


def layout(groups):
    """Rows of GROUPS_PER_ROW groups (zero-padded), and the inv_lambda vector: column block j of
    16 columns takes INV_LAMBDAS[j % 8]."""
    ng = groups.shape[0]
    rows = (ng + GROUPS_PER_ROW - 1) // GROUPS_PER_ROW
    flat = np.zeros((rows * GROUPS_PER_ROW, 16), dtype=np.uint16)
    flat[:ng] = groups
    Xb = flat.reshape(rows, K)
    il = np.repeat(INV_LAMBDAS[np.arange(GROUPS_PER_ROW) % len(INV_LAMBDAS)], 16)
    return Xb, il


WINDOWS = list(range(-116, 117, 16))  # -116, -100, ..., 108


def runs():
    """(s_x, value selection) per run: windows of 2^16 over [2^-116, 2^116], then one run of all
    values at s_x = 1."""
    out = []
    for i, e in enumerate(WINDOWS):
        s = 2.0 ** e * (1.37 if i % 2 else 1.0)
        s = min(max(s, 2.0 ** -116), 2.0 ** 116)
        out.append((float(np.float32(s)), e))
    out.append((1.0, None))
    return out


@pytest.fixture(scope="module")
def lib():
    from bit_rank_compensated_b200 import svdq

    svdq.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return svdq


def test_sweep_covers_every_finite_bf16_value():
    vb = finite_bf16_bits()
    assert vb.size == 65280
    mag = np.abs(bf16_bits_to_f32(vb).astype(np.float64))
    covered = np.zeros(vb.size, bool)
    for s, e in runs():
        if e is None:
            covered[:] = True
        else:
            lo, hi = 2.0 ** (e - 16), 2.0 ** (e + 16)
            covered |= (mag >= lo) & (mag <= hi)
    assert covered.all()


@pytest.mark.parametrize("s_x,e", runs(), ids=[f"s{i}" for i in range(len(runs()))])
def test_activation_codes_exhaustive(lib, s_x, e):
    rng = np.random.default_rng(abs(e or 0) + 7)
    vb = finite_bf16_bits()
    if e is not None:
        mag = np.abs(bf16_bits_to_f32(vb).astype(np.float64))
        keep = (mag >= 2.0 ** (e - 16)) & (mag <= 2.0 ** (e + 16))
        if e == WINDOWS[0]:
            keep |= mag < 2.0 ** (e - 16)  # the smallest values, subnormals and zero
        if e == WINDOWS[-1]:
            keep |= mag > 2.0 ** (e + 16)  # up to the largest finite bf16
        vb = vb[keep]
    groups = sweep_groups(vb, rng)
    Xb, il = layout(groups)
    M = Xb.shape[0]
    rank = 32 if e == WINDOWS[7] else 0  # the production template (with the down-projection) on one run
    N = 16
    L = lib.Layer.from_arrays(N=N, K=K, rank=rank, wq=np.zeros((N, K // 2), np.uint8),
                              ws=np.zeros(lib.weight_scale_bytes(N, K), np.uint8), inv_lambda=il,
                              L1t=np.zeros((rank, K), np.uint16) if rank else None,
                              L2t=np.zeros((N, rank), np.uint16) if rank else None, bias=None, s_w=1.0, s_x=s_x)
    xq, xs, _ = lib.quant_act_lora_down(x_to_device(Xb), L)
    torch.cuda.synchronize()
    assert lib.last_device_error() == 0
    Xh = O.f32(bf16_bits_to_f32(Xb).astype(np.float64) * il.astype(np.float64)[None, :])
    assert np.all(np.isfinite(Xh))
    codes, scales = O.nvfp4_quantize(Xh, s_x)
    got_c = xq.cpu().numpy().reshape(M, K // 2)
    want_c = O.pack_codes(codes)
    bad = np.argwhere(got_c != want_c)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:4].tolist()}"
    got_s = lib.unswizzle_scales(xs.cpu().numpy(), M, K)
    np.testing.assert_array_equal(got_s, scales)
