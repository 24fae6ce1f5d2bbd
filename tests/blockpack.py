"""Test-side block encoders: pack intended quantization parameters into canonical bytes.

These are the inverse of the block layouts (ds4 pages: up/gate IQ2_XXS-style,
down Q2_K-style, and the 4-bit Q4_K-style "q4" experts).  They are used to
hand-build blocks whose dequantized values are known exactly, independently
of any decoder.  They hold no decoding logic.
"""
import numpy as np


def f16_bits(v: float) -> int:
    return int(np.array([v], dtype=np.float16).view(np.uint16)[0])


def pack_iq2x(d_bits: int, idx, signs, scales) -> np.ndarray:
    """idx[8][4] grid indices, signs[8][4][8] in {0,1} (even parity per 8-vector), scales[8] in 0..15."""
    b = np.zeros(66, np.uint8)
    b[0] = d_bits & 0xFF
    b[1] = d_bits >> 8
    for g in range(8):
        base = 2 + 8 * g
        aux = int(scales[g]) << 28
        for j in range(4):
            b[base + j] = idx[g][j]
            sg = [int(v) for v in signs[g][j]]
            assert sum(sg) % 2 == 0, "IQ2X 8-vectors carry an even number of negatives"
            for i in range(7):
                aux |= sg[i] << (7 * j + i)
        for t in range(4):
            b[base + 4 + t] = (aux >> (8 * t)) & 0xFF
    return b


def pack_q2k(d_bits: int, dmin_bits: int, sc, m, q) -> np.ndarray:
    """sc[16], m[16] in 0..15, q[256] in 0..3."""
    b = np.zeros(84, np.uint8)
    for s in range(16):
        b[s] = (int(sc[s]) & 0xF) | ((int(m[s]) & 0xF) << 4)
    for i in range(256):
        b[16 + i // 4] |= (int(q[i]) & 3) << (2 * (i % 4))
    b[80], b[81] = d_bits & 0xFF, d_bits >> 8
    b[82], b[83] = dmin_bits & 0xFF, dmin_bits >> 8
    return b


def pack_q4k(d_bits: int, dmin_bits: int, sc, m, q) -> np.ndarray:
    """sc[8], m[8] in 0..63, q[256] in 0..15."""
    b = np.zeros(144, np.uint8)
    b[0], b[1] = d_bits & 0xFF, d_bits >> 8
    b[2], b[3] = dmin_bits & 0xFF, dmin_bits >> 8
    bits = 0
    for j in range(8):
        bits |= (int(sc[j]) & 63) << (6 * j)
        bits |= (int(m[j]) & 63) << (48 + 6 * j)
    for t in range(12):
        b[4 + t] = (bits >> (8 * t)) & 0xFF
    for i in range(256):
        b[16 + i // 2] |= (int(q[i]) & 15) << (4 * (i % 2))
    return b
