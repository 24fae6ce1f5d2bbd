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


def _top8(L, x):
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    logits = xf @ L.wr.view(np.float16).astype(np.float64).T + L.bias
    return np.argsort(-logits, axis=1, kind="stable")[:, :8]


def test_routing_skew_of_the_skewed_workloads():
    """The router bias N(0, 1) gives the skew the workloads describe: at T=4096 the busiest expert gets about 10x
    the mean load, and a batch of B tokens touches far fewer than 8 B distinct experts."""
    wl = synth.WORKLOADS["prefill"]
    counts = np.bincount(_top8(synth.make_layer(wl), synth.activations(wl, 4096)).ravel(), minlength=256)
    assert 10 <= counts.max() / counts.mean() <= 17
    wl = synth.WORKLOADS["batched"]
    L = synth.make_layer(wl)
    unique = []
    for B in (4, 16, 64):
        ids = _top8(L, synth.activations(wl, 8 * B, stream=40 + B)).reshape(8, B * 8)
        unique.append(np.mean([len(np.unique(r)) for r in ids]))
    assert 8 < unique[0] < unique[1] < unique[2] < 0.5 * 8 * 64
