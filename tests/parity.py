"""Comparison rules between the CUDA path and the oracle.

Criteria (the layer's acceptance bar): dequantized weights bit-exact; top-k ids
equal wherever the oracle's k-th score gap exceeds 1e-4; layer output within
relative L2 <= 5e-3 and max-abs <= 2e-2 * rms(oracle output).  Where a token's
gap is <= 1e-4 both the oracle's selection and the alternative with ranks k and
k+1 swapped are correct; the GPU must pick one of them and its output is
compared with the oracle's output for that selection.
"""
import numpy as np

import oracle

GAP_TOL = 1e-4
REL_L2 = 5e-3
MAX_ABS_RMS = 2e-2


def bf16_bits_to_f64(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_tensor_to_f64(t):
    import torch
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16).astype(np.uint32).__lshift__(16) \
        .view(np.float32).astype(np.float64)


def oracle_layer(L, x, nthreads=None):
    """Oracle outputs for both the normal and the alternative selection."""
    args = (L.shape, x, L.wr, L.bias, L.grid, L.expert, (L.sh_gate, L.sh_up, L.sh_down))
    out0, ids0, w0, gap = oracle.layer_forward(*args, alt=False, nthreads=nthreads)
    near = gap <= GAP_TOL
    out1 = ids1 = None
    if np.any(near):
        sub = np.nonzero(near)[0]
        o1, i1, _, _ = oracle.layer_forward(L.shape, x[sub], L.wr, L.bias, L.grid, L.expert,
                                            (L.sh_gate, L.sh_up, L.sh_down), alt=True, nthreads=nthreads)
        out1 = dict(zip(sub.tolist(), o1))
        ids1 = dict(zip(sub.tolist(), i1))
    return dict(out=out0, ids=ids0, w=w0, gap=gap, near=near, out_alt=out1, ids_alt=ids1)


def check_ids(gpu_ids, ref):
    """Returns the per-token oracle output to compare against; asserts the id rule."""
    ids0, near = ref["ids"], ref["near"]
    want = ref["out"].copy()
    n_near_alt = 0
    for t in range(ids0.shape[0]):
        g = [int(v) for v in gpu_ids[t]]
        if not near[t]:
            assert g == ids0[t].tolist(), "token %d: ids %s != oracle %s (gap %.3g)" % (t, g, ids0[t].tolist(),
                                                                                        ref["gap"][t])
        else:
            alt = ref["ids_alt"][t].tolist()
            assert g in (ids0[t].tolist(), alt), "token %d: near-tie ids %s not in {%s, %s}" % (
                t, g, ids0[t].tolist(), alt)
            if g == alt and g != ids0[t].tolist():
                want[t] = ref["out_alt"][t]
                n_near_alt += 1
    return want, n_near_alt


def output_errors(gpu, want):
    err = gpu - want
    rel = np.linalg.norm(err) / max(np.linalg.norm(want), 1e-300)
    rms = np.sqrt(np.mean(want ** 2))
    mx = np.abs(err).max() / max(rms, 1e-300)
    return rel, mx


def assert_output_close(gpu, want, what=""):
    rel, mx = output_errors(gpu, want)
    assert rel <= REL_L2, "%s rel L2 %.3g > %.1g" % (what, rel, REL_L2)
    assert mx <= MAX_ABS_RMS, "%s max-abs %.3g rms > %.1g" % (what, mx, MAX_ABS_RMS)
    return rel, mx
