"""The seeded generators: determinism and the value distributions the workloads state."""
import numpy as np

from bit_quantized_moe_02_b200 import synth


def test_codebook_values_and_determinism():
    g = synth.codebook(0)
    assert g.shape == (256, 8) and set(np.unique(g)) <= {8, 25, 43}
    assert np.array_equal(g, synth.codebook(0)) and not np.array_equal(g, synth.codebook(1))


def test_block_scales_are_abs_normal_fp16():
    for fmt, offs in (("iq2x", (0,)), ("q2k", (80, 82)), ("q4k", (0, 2))):
        b = synth.random_blocks(fmt, 4096, synth.rng(1, 2, 3))
        for o in offs:
            d = (b[:, o].astype(np.uint16) | (b[:, o + 1].astype(np.uint16) << 8)).view(np.float16)
            d = d.astype(np.float64)
            assert np.all(d >= 0) and np.all(np.isfinite(d))
            assert abs(d.mean() - 1e-3 * np.sqrt(2 / np.pi)) < 5e-5


def test_layer_is_reproducible_per_expert():
    wl = synth.WORKLOADS["tiny"]
    a, b = synth.make_layer(wl), synth.make_layer(wl)
    assert np.array_equal(a.wr, b.wr) and np.array_equal(a.expert("down", 5), b.expert("down", 5))
    assert a.expert("gate", 0).shape == (512, 66)
    assert a.expert("down", 0).shape == (256, 2 * 84)
    assert np.all(a.bias == 0)
    x = synth.activations(wl, 3)
    assert x.shape == (3, 256) and x.dtype == np.uint16


def test_bf16_rounding_nearest_even():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -2.5], np.float32)
    bits = synth.f32_to_bf16_bits(v)
    back = (bits.astype(np.uint32) << 16).view(np.float32)
    assert back.tolist() == [1.0, 1.0, 1.0 + 2 ** -7, -2.5]
