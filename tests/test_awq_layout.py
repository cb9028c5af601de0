"""CPU check of the awq_w4a16 GEMV's data path (tests/awq_layout.py): the tile layout the pack
kernel writes and the staged activations, placed in m16n8k16 MMA fragments as the PTX ISA
defines them, reproduce the oracle's dequantized product."""
import numpy as np

from oracle import svdq_oracle as O
def test_tile_layout_feeds_the_mma_fragments():
    # the GEMV's data path on the CPU: packed tiles and staged activations through the m16n8k16
    # fragment placement give the oracle's dequantized product
    from synth import bf16_bits_to_f32, make_modulation_inputs
    from tests.awq_layout import emulate_gemv

    Xb, W, _ = make_modulation_inputs(3, 128, 21, seed=3)
    X = bf16_bits_to_f32(Xb).astype(np.float64)
    q, s, z = O.awq_quantize(W)
    s16 = s.astype(np.float16).astype(np.float64)
    got = emulate_gemv(X, q, s16, z)
    want = O.awq_linear(X, q, s, z)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
