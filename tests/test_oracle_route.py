"""Pins of the oracle's router: closed forms, invariants and an independent numpy recomputation.

Router left unquantized (ds4 news summary, "model weights"); gating = sigmoid
scores, top-k, renormalised to sum 1.  Bias is added to the logit before the
sigmoid; ties go to the smaller expert id.
"""
import math

import numpy as np
import pytest

import oracle
from bit_quantized_moe_02_b200 import synth


def _f16(a):
    return np.asarray(a, np.float32).astype(np.float16).view(np.uint16)


def _bf16(a):
    return synth.f32_to_bf16_bits(np.asarray(a, np.float32))


def sig(v):
    return 1.0 / (1.0 + math.exp(-v))


def test_two_expert_closed_form():
    d = 256
    x = np.zeros((1, d), np.float32)
    x[0, 3] = 2.0
    wr = np.zeros((2, d), np.float32)
    wr[0, 3] = 0.25    # logit 0.5
    wr[1, 3] = -0.125  # logit -0.25, +bias 0.25 -> 0
    bias = np.array([0.0, 0.25], np.float32)
    ids, w, scores, gap = oracle.route(_bf16(x), _f16(wr), bias, k=2)
    s0, s1 = sig(0.5), sig(0.0)
    assert ids.tolist() == [[0, 1]]
    assert scores[0, 0] == pytest.approx(s0, abs=1e-15) and scores[0, 1] == pytest.approx(0.5, abs=1e-15)
    assert w[0, 0] == pytest.approx(s0 / (s0 + s1), abs=1e-15)
    assert w[0, 1] == pytest.approx(s1 / (s0 + s1), abs=1e-15)
    ids, w, _, gap = oracle.route(_bf16(x), _f16(wr), bias, k=1)
    assert ids.tolist() == [[0]] and w[0, 0] == 1.0 and gap[0] == pytest.approx(s0 - s1, abs=1e-15)


def test_bias_enters_before_sigmoid():
    d, E = 256, 5
    x = np.zeros((1, d), np.float32)
    bias = np.array([-1.0, 2.0, 0.5, 0.0, 1.0], np.float32)
    _, _, scores, _ = oracle.route(_bf16(x), _f16(np.zeros((E, d))), bias, k=2)
    assert np.allclose(scores[0], [sig(b) for b in bias], atol=1e-15, rtol=0)


def test_ties_go_to_smaller_id():
    d, E = 256, 6
    x = _bf16(np.random.default_rng(0).normal(size=(1, d)))
    row = np.random.default_rng(1).normal(0, 0.02, size=d)
    wr = _f16(np.stack([row] * E))
    ids, w, _, gap = oracle.route(x, wr, None, k=3)
    assert ids.tolist() == [[0, 1, 2]]
    assert gap[0] == 0.0
    assert np.allclose(w, 1.0 / 3.0, atol=1e-15)


def test_invariants_and_numpy_recomputation():
    r = np.random.default_rng(3)
    T, d, E, k = 37, 512, 64, 6
    x = _bf16(r.normal(size=(T, d)))
    wr = _f16(r.normal(0, 0.02, size=(E, d)))
    bias = r.normal(0, 1, size=E).astype(np.float32)
    ids, w, scores, gap = oracle.route(x, wr, bias, k)
    # independent recomputation with numpy float64 (library matmul)
    xf = x.astype(np.uint32) << 16
    xf = xf.view(np.float32).astype(np.float64)
    wf = wr.view(np.float16).astype(np.float64)
    logit = xf @ wf.T + bias.astype(np.float64)
    s = 1.0 / (1.0 + np.exp(-logit))
    assert np.allclose(scores, s, rtol=0, atol=1e-13)
    order = np.lexsort((np.arange(E)[None, :].repeat(T, 0), -s), axis=1)
    assert np.array_equal(ids, order[:, :k].astype(np.int32))
    for t in range(T):
        assert len(set(ids[t])) == k
        ss = s[t, ids[t]]
        assert np.all(np.diff(ss) <= 0)
        assert gap[t] == pytest.approx(ss[-1] - np.sort(s[t])[::-1][k], abs=1e-13)
    assert np.all(w > 0)
    assert np.allclose(w.sum(1), 1.0, atol=1e-12, rtol=0)


def test_k_equals_E_selects_all():
    r = np.random.default_rng(4)
    d, E = 256, 8
    ids, w, scores, _ = oracle.route(_bf16(r.normal(size=(3, d))), _f16(r.normal(0, .02, (E, d))), None, k=E)
    for t in range(3):
        assert sorted(ids[t].tolist()) == list(range(E))
        assert np.allclose(w[t], scores[t, ids[t]] / scores[t].sum(), atol=1e-15)


def test_alt_swaps_kth_and_next():
    r = np.random.default_rng(5)
    d, E, k = 256, 16, 4
    x = _bf16(r.normal(size=(5, d)))
    wr = _f16(r.normal(0, .05, (E, d)))
    ids, _, scores, _ = oracle.route(x, wr, None, k)
    ids_alt, w_alt, _, _ = oracle.route(x, wr, None, k, alt=True)
    for t in range(5):
        full = np.lexsort((np.arange(E), -scores[t]))
        assert ids[t].tolist() == full[:k].tolist()
        assert ids_alt[t].tolist() == full[:k - 1].tolist() + [full[k]]
        assert w_alt[t].sum() == pytest.approx(1.0, abs=1e-12)
