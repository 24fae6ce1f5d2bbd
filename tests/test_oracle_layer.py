"""Pins of the oracle's whole layer: hand cases and an independent dense numpy float64 brute force.

The brute force rebuilds every matrix densely from the (separately pinned)
block dequantization and runs the layer with numpy matmuls, so a dropped term,
wrong index or transposed operand in the oracle's contraction, SwiGLU, gating
or combine fails here.
"""
import dataclasses

import numpy as np
import pytest

import oracle
from bit_quantized_moe_02_b200 import synth


def bf16_to_f64(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def tiny_layer(E=4, k=2, d=256, f=256, fs=256, bias_std=1.0, seed=11, fmts=("iq2x", "iq2x", "q2k")):
    shape = synth.LayerShape(d=d, E=E, f=f, k=k, f_shared=fs, fmt_gate=fmts[0], fmt_up=fmts[1], fmt_down=fmts[2])
    wl = synth.Workload("t", shape, (1,), bias_std, seed)
    return synth.make_layer(wl)


def dense(L, which, e):
    s = L.shape
    fmt = {"gate": s.fmt_gate, "up": s.fmt_up, "down": s.fmt_down}[which]
    rows, cols = (s.d, s.f) if which == "down" else (s.f, s.d)
    return oracle.dequant(fmt, L.expert(which, e), L.grid).astype(np.float64).reshape(rows, cols)


def numpy_layer(L, x_bits):
    s = L.shape
    x = bf16_to_f64(x_bits)
    wr = L.wr.view(np.float16).astype(np.float64)
    sc = 1.0 / (1.0 + np.exp(-(x @ wr.T + L.bias.astype(np.float64))))
    out = np.zeros((x.shape[0], s.d))
    if s.f_shared:
        g = x @ bf16_to_f64(L.sh_gate).T
        u = x @ bf16_to_f64(L.sh_up).T
        out += (g / (1 + np.exp(-g)) * u) @ bf16_to_f64(L.sh_down).T
    for t in range(x.shape[0]):
        ids = np.lexsort((np.arange(s.E), -sc[t]))[:s.k]
        w = sc[t, ids] / sc[t, ids].sum()
        for j, e in enumerate(ids):
            g = dense(L, "gate", e) @ x[t]
            u = dense(L, "up", e) @ x[t]
            out[t] += w[j] * (dense(L, "down", e) @ (g / (1 + np.exp(-g)) * u))
    return out


def run_oracle(L, x, alt=False, nthreads=2):
    return oracle.layer_forward(L.shape, x, L.wr, L.bias, L.grid, L.expert, (L.sh_gate, L.sh_up, L.sh_down),
                                alt=alt, nthreads=nthreads)


@pytest.mark.parametrize("fmts", [("iq2x", "iq2x", "q2k"), ("q4k", "q4k", "q4k")])
def test_brute_force_dense_numpy(fmts):
    L = tiny_layer(fmts=fmts)
    x = synth.f32_to_bf16_bits(np.random.default_rng(2).normal(size=(5, 256)).astype(np.float32))
    out, ids, w, gap = run_oracle(L, x)
    ref = numpy_layer(L, x)
    assert np.allclose(out, ref, rtol=1e-11, atol=1e-13 * np.abs(ref).max())


def test_brute_force_larger_dims_no_shared():
    L = tiny_layer(E=6, k=3, d=512, f=768, fs=0, seed=5)
    x = synth.f32_to_bf16_bits(np.random.default_rng(8).normal(size=(3, 512)).astype(np.float32))
    out, _, _, _ = run_oracle(L, x, nthreads=3)
    ref = numpy_layer(L, x)
    assert np.allclose(out, ref, rtol=1e-11, atol=1e-13 * np.abs(ref).max())


def test_zero_input_gives_zero_output():
    L = tiny_layer()
    out, ids, w, _ = run_oracle(L, np.zeros((2, 256), np.uint16))
    assert np.all(out == 0.0)
    # zero logits + bias: all scores sigma(bias); weights renormalised over the chosen ones
    assert np.allclose(w.sum(1), 1.0, atol=1e-14)


def test_single_expert_weight_one_equals_its_ffn():
    L = tiny_layer(E=1, k=1, fs=0)
    x = synth.f32_to_bf16_bits(np.random.default_rng(4).normal(size=(1, 256)).astype(np.float32))
    out, ids, w, _ = run_oracle(L, x)
    assert ids.tolist() == [[0]] and w[0, 0] == 1.0
    xv = bf16_to_f64(x[0])
    g, u = dense(L, "gate", 0) @ xv, dense(L, "up", 0) @ xv
    y = dense(L, "down", 0) @ (g / (1 + np.exp(-g)) * u)
    assert np.allclose(out[0], y, rtol=1e-12, atol=1e-14)


def test_unit_vector_input_reads_one_column():
    # x = e_i: g = G[:, i], u = U[:, i] exactly; check h through the down matrix.
    L = tiny_layer(E=1, k=1, fs=0)
    x = np.zeros((1, 256), np.uint16)
    x[0, 17] = synth.f32_to_bf16_bits(np.array([1.0], np.float32))[0]
    out, _, _, _ = run_oracle(L, x)
    g, u = dense(L, "gate", 0)[:, 17], dense(L, "up", 0)[:, 17]
    h = g * (1 / (1 + np.exp(-g))) * u
    assert np.allclose(out[0], dense(L, "down", 0) @ h, rtol=1e-12, atol=1e-15)


def test_alt_selection_changes_only_kth_expert():
    L = tiny_layer(E=4, k=2)
    x = synth.f32_to_bf16_bits(np.random.default_rng(9).normal(size=(4, 256)).astype(np.float32))
    out0, ids0, _, _ = run_oracle(L, x)
    out1, ids1, _, _ = run_oracle(L, x, alt=True)
    assert np.array_equal(ids0[:, 0], ids1[:, 0])
    assert np.all(ids0[:, 1] != ids1[:, 1])
    assert not np.allclose(out0, out1)


def test_threads_do_not_change_result():
    L = tiny_layer()
    x = synth.f32_to_bf16_bits(np.random.default_rng(10).normal(size=(7, 256)).astype(np.float32))
    a = run_oracle(L, x, nthreads=1)[0]
    b = run_oracle(L, x, nthreads=4)[0]
    assert np.array_equal(a, b)
