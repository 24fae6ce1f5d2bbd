"""Pins of the oracle's block dequantization against closed forms and hand-packed blocks.

Formats: IQ2_XXS-style up/gate and Q2_K-style down (ds4 news summary, "model
weights"; upppp.jp, "asymmetric 2-bit quantization"), Q4_K-style 4-bit
experts (ds4 news summary, "speed benchmarks", q4 model).  Every expected
value below is exact in fp32, so equality is required.
"""
import itertools

import numpy as np
import pytest

import oracle
from tests.blockpack import f16_bits, pack_iq2x, pack_q2k, pack_q4k

F16 = np.float16


def grid_const(v=8):
    return np.full((256, 8), v, np.uint8)


def test_f16_decoding_matches_numpy_all_finite_patterns():
    # Constant Q2K blocks with sc=1, q=1, m=0 give w = d exactly, for every finite fp16 pattern d.
    pats = np.arange(0, 0x7C00, dtype=np.uint16)  # +0 .. max finite, incl. subnormals
    blocks = np.stack([pack_q2k(int(p), 0, [1] * 16, [0] * 16, [1] * 256) for p in pats[::97]] +
                      [pack_q2k(int(p), 0, [1] * 16, [0] * 16, [1] * 256) for p in (1, 0x3FF, 0x400, 0x7BFF)])
    w = oracle.dequant("q2k", blocks).reshape(len(blocks), 256)
    want = np.concatenate([pats[::97], np.array([1, 0x3FF, 0x400, 0x7BFF], np.uint16)]).view(F16).astype(np.float32)
    assert np.array_equal(w, np.repeat(want[:, None], 256, axis=1))


def test_iq2x_closed_form_all_eights_max_scale():
    # grid entry 0 = all 8, no negatives, s = 15 -> w = d * 15.5 * 0.25 * 8 = 31 d for all 256 weights.
    d = 0.00123
    b = pack_iq2x(f16_bits(d), [[0] * 4] * 8, [[[0] * 8] * 4] * 8, [15] * 8)
    w = oracle.dequant("iq2x", b, grid_const(8))
    assert np.array_equal(w, np.full(256, 31.0 * float(F16(d)), np.float32))


def test_iq2x_scale_zero_is_grid_over_eight():
    d = 0.75
    grid = np.zeros((256, 8), np.uint8)
    grid[7] = [8, 25, 43, 8, 25, 43, 8, 25]
    b = pack_iq2x(f16_bits(d), [[7] * 4] * 8, [[[0] * 8] * 4] * 8, [0] * 8)
    w = oracle.dequant("iq2x", b, grid)
    want = np.tile(np.array(grid[7], np.float64) * float(F16(d)) / 8.0, 32).astype(np.float32)
    assert np.array_equal(w, want)


@pytest.mark.parametrize("g,j,i", [(0, 0, 0), (3, 2, 5), (7, 3, 6), (5, 1, 3)])
def test_iq2x_single_sign_bit_flips_element_and_parity_partner(g, j, i):
    # Setting stored sign bit i of vector j negates element i and, through parity, element 7.
    grid = grid_const(25)
    signs = [[[0] * 8 for _ in range(4)] for _ in range(8)]
    signs[g][j][i] = 1
    signs[g][j][7] = 1
    b = pack_iq2x(f16_bits(1.0), [[0] * 4] * 8, signs, [3] * 8)
    w = oracle.dequant("iq2x", b, grid)
    mag = 1.0 * 3.5 * 0.25 * 25
    want = np.full(256, mag, np.float32)
    want[32 * g + 8 * j + i] = -mag
    want[32 * g + 8 * j + 7] = -mag
    assert np.array_equal(w, want)


def test_iq2x_random_params_pin_layout():
    r = np.random.default_rng(7)
    grid = np.asarray([8, 25, 43], np.uint8)[r.integers(0, 3, (256, 8))]
    for trial in range(20):
        d = float(F16(abs(r.normal(0, 1e-2)) + 1e-5))
        idx = r.integers(0, 256, (8, 4))
        signs = r.integers(0, 2, (8, 4, 8))
        signs[:, :, 7] = signs[:, :, :7].sum(-1) % 2
        scales = r.integers(0, 16, 8)
        b = pack_iq2x(f16_bits(d), idx.tolist(), signs.tolist(), scales.tolist())
        w = oracle.dequant("iq2x", b, grid)
        want = np.empty(256)
        for g, j, i in itertools.product(range(8), range(4), range(8)):
            want[32 * g + 8 * j + i] = (d * (0.5 + scales[g]) * 0.25 * grid[idx[g, j], i] *
                                       (-1.0 if signs[g, j, i] else 1.0))
        assert np.array_equal(w, want.astype(np.float32)), trial  # exact: <= 22 significant bits


def test_q2k_closed_forms():
    d, dmin = 0.0625, 0.001953125
    w = oracle.dequant("q2k", pack_q2k(f16_bits(d), f16_bits(dmin), [1] * 16, [0] * 16, [3] * 256))
    assert np.array_equal(w, np.full(256, 3 * d, np.float32))
    w = oracle.dequant("q2k", pack_q2k(f16_bits(d), f16_bits(dmin), [5] * 16, [1] * 16, [0] * 256))
    assert np.array_equal(w, np.full(256, -dmin, np.float32))


def test_q2k_single_weight_every_position():
    d = 0.5
    blocks = []
    for p in range(256):
        q = [0] * 256
        q[p] = 2
        sc = [0] * 16
        sc[p // 16] = 3
        blocks.append(pack_q2k(f16_bits(d), f16_bits(0.25), sc, [0] * 16, q))
    w = oracle.dequant("q2k", np.stack(blocks)).reshape(256, 256)
    assert np.array_equal(w, np.eye(256, dtype=np.float32) * (d * 3 * 2))


def test_q2k_scale_min_nibbles_per_subblock():
    d, dmin = 0.125, 0.0078125
    sc = list(range(16))
    m = [15 - s for s in range(16)]
    w = oracle.dequant("q2k", pack_q2k(f16_bits(d), f16_bits(dmin), sc, m, [1] * 256))
    want = np.repeat([d * sc[s] - dmin * m[s] for s in range(16)], 16).astype(np.float32)
    assert np.array_equal(w, want)


def test_q4k_single_weight_every_position():
    d = 0.25
    blocks = []
    for p in range(256):
        q = [0] * 256
        q[p] = 9
        sc = [0] * 8
        sc[p // 32] = 37
        blocks.append(pack_q4k(f16_bits(d), f16_bits(0.5), sc, [0] * 8, q))
    w = oracle.dequant("q4k", np.stack(blocks)).reshape(256, 256)
    assert np.array_equal(w, np.eye(256, dtype=np.float32) * (d * 37 * 9))


def test_q4k_six_bit_fields():
    d, dmin = 0.015625, 0.0009765625
    sc = [1, 63, 17, 42, 5, 33, 60, 2]
    m = [63, 0, 31, 8, 50, 12, 1, 44]
    q = [(i * 7) % 16 for i in range(256)]
    w = oracle.dequant("q4k", pack_q4k(f16_bits(d), f16_bits(dmin), sc, m, q))
    want = np.array([d * sc[i // 32] * q[i] - dmin * m[i // 32] for i in range(256)])
    # single rounding (the subtraction) on exact products
    assert np.array_equal(w, want.astype(np.float32))


@pytest.mark.parametrize("fmt", ["q2k", "q4k"])
def test_k_formats_special_d_values(fmt):
    # fp16 subnormal, zero and max d with dmin = 0: w = d * sc * q exactly.
    for dbits in (0x0001, 0x0000, 0x7BFF, 0x03FF):
        dv = float(np.array([dbits], np.uint16).view(F16)[0])
        if fmt == "q2k":
            b = pack_q2k(dbits, 0, [2] * 16, [0] * 16, [3] * 256)
            want = dv * 2 * 3
        else:
            b = pack_q4k(dbits, 0, [2] * 8, [0] * 8, [15] * 256)
            want = dv * 2 * 15
        assert np.array_equal(oracle.dequant(fmt, b), np.full(256, want, np.float32))
