"""CUDA path vs the oracle, through the C ABI (libds4moe.so), on seeded synthetic inputs.

Dequantization must be bit-exact; ids must match wherever the oracle's k-th
score gap exceeds 1e-4; outputs must be within rel-L2 5e-3 and max-abs
2e-2 * rms of the oracle's fp64 result.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from bit_quantized_moe_02_b200 import synth
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ds4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_moe_02_b200 import ds4moe
    ds4moe.lib()
    return ds4moe


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def layer_of(shape, bias_std, seed):
    return synth.make_layer(synth.Workload("test", shape, (1,), bias_std, seed))


# ---------------------------------------------------------------------------------------------------------
# dequantization: bit-exact


@pytest.mark.parametrize("fmt,rows,cols", [("iq2x", 37, 512), ("iq2x", 4, 4096), ("q2k", 33, 768),
                                           ("q2k", 8, 2048), ("q4k", 19, 1024)])
def test_dequant_bit_exact(ds4, fmt, rows, cols):
    g = synth.rng(99, rows, cols)
    canon = synth.random_matrix(fmt, rows, cols, g)
    # plant special scales: fp16 subnormal, zero and max d in the first blocks
    offs = {"iq2x": (0,), "q2k": (80, 82), "q4k": (0, 2)}[fmt]
    flat = canon.reshape(-1, synth.BLOCK_BYTES[fmt])
    for i, bits in enumerate((0x0001, 0x0000, 0x7BFF, 0x03FF)):
        for o in offs:
            flat[i, o], flat[i, o + 1] = bits & 0xFF, bits >> 8
    grid = synth.codebook(5)
    want = oracle.dequant(fmt, canon, grid if fmt == "iq2x" else None).reshape(rows, cols)
    prep = ds4.prepare(fmt, dev(canon), rows, cols, 1)
    got = ds4.dequant(fmt, prep, dev(grid.reshape(-1)) if fmt == "iq2x" else None, rows, cols).cpu().numpy()
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_prepare_many_matrices_with_stride(ds4):
    rows, cols, n = 16, 512, 5
    mats = np.stack([synth.random_matrix("iq2x", rows, cols, synth.rng(7, m)) for m in range(n)])
    grid = synth.codebook(3)
    prep = ds4.prepare("iq2x", dev(mats), rows, cols, n)
    stride = prep.numel() // n
    for m in range(n):
        got = ds4.dequant("iq2x", prep[m * stride:], dev(grid.reshape(-1)), rows, cols).cpu().numpy()
        assert np.array_equal(got, oracle.dequant("iq2x", mats[m], grid).reshape(rows, cols))


# ---------------------------------------------------------------------------------------------------------
# router


@pytest.mark.parametrize("T,d,E,k,bias_std", [(1, 256, 8, 2, 0.0), (1, 4096, 256, 8, 0.0), (5, 4096, 256, 8, 1.0),
                                              (300, 1024, 64, 6, 1.0), (130, 4096, 256, 8, 1.0)])
def test_route_matches_oracle(ds4, T, d, E, k, bias_std):
    g = synth.rng(5, T, d, E)
    x = synth.f32_to_bf16_bits(g.normal(size=(T, d)).astype(np.float32))
    wr = synth.f32_to_f16_bits(g.normal(0, 0.02, size=(E, d)).astype(np.float32))
    bias = g.normal(0, bias_std, size=E).astype(np.float32) if bias_std else None
    ids0, w0, _, gap = oracle.route(x, wr, bias, k)
    ids, w = ds4.route(dev(x), dev(wr).view(torch.float16), dev(bias) if bias is not None else None, k)
    ids, w = ids.cpu().numpy(), w.cpu().numpy()
    far = gap > parity.GAP_TOL
    assert np.array_equal(ids[far], ids0[far])
    assert np.allclose(w[far], w0[far], atol=2e-6, rtol=0)
    assert np.allclose(w.sum(1), 1.0, atol=1e-5)
    for t in range(T):
        assert len(set(ids[t].tolist())) == k


def test_route_ties_to_smaller_id(ds4):
    d, E, k = 256, 16, 4
    x = synth.f32_to_bf16_bits(np.ones((1, d), np.float32))
    wr = np.zeros((E, d), np.float32)
    wr[[3, 7, 9, 12, 14]] = 0.01
    ids, _ = ds4.route(dev(x), dev(synth.f32_to_f16_bits(wr)).view(torch.float16), None, k)
    assert ids.cpu().numpy().tolist() == [[3, 7, 9, 12]]


# ---------------------------------------------------------------------------------------------------------
# whole layer


def run_and_compare(ds4, L, x, path, nthreads=None):
    D = ds4.DeviceLayer(L, max_tokens=x.shape[0])
    xt = dev(x).view(torch.bfloat16)
    if path == "decode":
        outs, idss = [], []
        for t in range(x.shape[0]):  # B = 1 decode per token
            o, ids, _ = D.forward(xt[t:t + 1], return_routing=True)
            outs.append(o)
            idss.append(ids)
        out, ids = torch.cat(outs), torch.cat(idss)
    elif path == "batched":
        out, ids, _ = D.forward(xt, return_routing=True)
    elif path == "fused":
        out, ids, _ = D.forward_fused(xt)
    else:
        out, ids, _, _, _ = D.forward_grouped(xt)
    torch.cuda.synchronize()
    assert ds4.last_device_error() == 0
    gpu = out.double().cpu().numpy()
    ref = parity.oracle_layer(L, x, nthreads=nthreads)
    want, _ = parity.check_ids(ids.cpu().numpy(), ref)
    return parity.assert_output_close(gpu, want, path)


def test_tiny_decode(ds4):
    wl = synth.WORKLOADS["tiny"]
    L = synth.make_layer(wl)
    x = synth.activations(wl, 6)
    run_and_compare(ds4, L, x, "decode")


@pytest.mark.parametrize("path", ["grouped", "fused"])
def test_tiny_grouped(ds4, path):
    wl = synth.WORKLOADS["tiny"]
    L = synth.make_layer(wl)
    x = synth.activations(wl, 150)
    run_and_compare(ds4, L, x, path)


@pytest.mark.parametrize("fs", [512, 0])
def test_fused_combine_matches_deterministic(ds4, fs):
    """The fused-combine prefill adds the k weighted rows of a token by atomic adds; it must agree with the
    deterministic grouped + combine path up to fp32 summation order (with and without a shared expert, whose
    absence makes the fused call zero the output first), and with the oracle at the layer tolerance."""
    shape = synth.LayerShape(d=1024, E=16, f=768, k=6, f_shared=fs)
    L = layer_of(shape, 1.0, 91 + fs)
    x = synth.f32_to_bf16_bits(synth.rng(9, fs).normal(size=(300, shape.d)).astype(np.float32))
    D = ds4.DeviceLayer(L, max_tokens=x.shape[0])
    xt = dev(x).view(torch.bfloat16)
    ref_out, ref_ids, ref_w, _, _ = D.forward_grouped(xt)
    out = torch.full((x.shape[0], shape.d), float("nan"), dtype=torch.float32, device="cuda")
    got, ids, w = D.forward_fused(xt, out=out)
    torch.cuda.synchronize()
    assert ds4.last_device_error() == 0
    assert got.data_ptr() == out.data_ptr()
    assert torch.equal(ids, ref_ids) and torch.equal(w, ref_w)
    a, b = got.double().cpu().numpy(), ref_out.double().cpu().numpy()
    assert np.all(np.isfinite(a))
    # k + 1 fp32 terms per element: reordering moves the sum by a few ulps of the largest partial sum
    assert np.max(np.abs(a - b)) <= 1e-5 * np.max(np.abs(b))
    run_and_compare(ds4, L, x, "fused")


@pytest.mark.parametrize("d,f,fs,E,k", [(512, 1024, 512, 16, 4), (1024, 256, 0, 12, 3), (2048, 512, 256, 32, 8)])
def test_mid_shapes_decode_and_grouped(ds4, d, f, fs, E, k):
    shape = synth.LayerShape(d=d, E=E, f=f, k=k, f_shared=fs)
    L = layer_of(shape, 1.0, 21 + d + f)
    x = synth.f32_to_bf16_bits(synth.rng(3, d, f).normal(size=(200, d)).astype(np.float32))
    run_and_compare(ds4, L, x[:4], "decode")
    run_and_compare(ds4, L, x, "grouped")  # several token tiles, ragged tail
    run_and_compare(ds4, L, x, "fused")


@pytest.mark.parametrize("d,f,fs,E,k", [(2048, 512, 1024, 16, 4), (4096, 1024, 2048, 16, 8)])
def test_decode_gemv_shapes(ds4, d, f, fs, E, k):
    """Single-token decode at the model's d with smaller f and E: other lane-slice widths of both GEMV kernels."""
    shape = synth.LayerShape(d=d, E=E, f=f, k=k, f_shared=fs)
    L = layer_of(shape, 1.0, 41 + f)
    x = synth.f32_to_bf16_bits(synth.rng(6, d, f).normal(size=(3, d)).astype(np.float32))
    run_and_compare(ds4, L, x, "decode")


@pytest.mark.parametrize("d,f,fs,E,k,fmt", [(1024, 4096, 512, 16, 4, "iq2x"), (1024, 512, 256, 32, 12, "iq2x"),
                                              (1024, 4096, 512, 16, 4, "q4k")])
def test_decode_gemv_one_warp_staging(ds4, d, f, fs, E, k, fmt):
    """Single-token decode where the down kernel stages each expert's h with one warp (f > 2048, or k > 8 experts,
    so two warps per expert do not fit): the other staging path of the GEMV down kernel."""
    f3 = {"fmt_gate": "q4k", "fmt_up": "q4k", "fmt_down": "q4k"} if fmt == "q4k" else {}
    shape = synth.LayerShape(d=d, E=E, f=f, k=k, f_shared=fs, **f3)
    L = layer_of(shape, 1.0, 51 + f + k)
    x = synth.f32_to_bf16_bits(synth.rng(9, d, f, k).normal(size=(2, d)).astype(np.float32))
    run_and_compare(ds4, L, x, "decode")


@pytest.mark.parametrize("d,f,fs,E,k", [(4096, 2048, 2048, 16, 8), (2048, 1024, 512, 16, 4), (1024, 256, 0, 8, 2)])
def test_q4k_decode_gemv(ds4, d, f, fs, E, k):
    """Single-token decode of Q4K layers through the GEMV kernels (the decode layer's shape with 16 experts, then
    smaller lane slices: 32 and 8 weights per lane in the down kernel, 4 and 2 vectors per lane in gate/up)."""
    shape = synth.LayerShape(d=d, E=E, f=f, k=k, f_shared=fs, fmt_gate="q4k", fmt_up="q4k", fmt_down="q4k")
    L = layer_of(shape, 1.0, 81 + d)
    x = synth.f32_to_bf16_bits(synth.rng(8, d).normal(size=(4, d)).astype(np.float32))
    run_and_compare(ds4, L, x, "decode")
    run_and_compare(ds4, L, x, "batched")  # B = 4: token by token through the same kernels


def test_q4k_layer_small(ds4):
    shape = synth.LayerShape(d=512, E=8, f=768, k=2, f_shared=256, fmt_gate="q4k", fmt_up="q4k", fmt_down="q4k")
    L = layer_of(shape, 1.0, 77)
    x = synth.f32_to_bf16_bits(synth.rng(4).normal(size=(70, 512)).astype(np.float32))
    run_and_compare(ds4, L, x, "grouped")
    run_and_compare(ds4, L, x, "fused")
    run_and_compare(ds4, L, x[:2], "decode")


@pytest.fixture(scope="module")
def decode_layer(ds4):
    wl = synth.WORKLOADS["decode"]
    return wl, synth.make_layer(wl)


def test_decode_full_size(ds4, decode_layer):
    wl, L = decode_layer
    x = synth.activations(wl, 8)
    run_and_compare(ds4, L, x, "decode")


@pytest.mark.parametrize("B", [2, 3, 4, 16, 17, 64])
def test_batched_decode(ds4, B):
    """B <= 16 runs the single-token GEMV pair token by token, larger batches the grouped path (17 and 64)."""
    wl = synth.WORKLOADS["batched"]
    L = synth.make_layer(wl)
    x = synth.activations(wl, B)
    run_and_compare(ds4, L, x, "batched")


@pytest.mark.parametrize("shape", [synth.WORKLOADS["tiny"].shape,
                                   synth.LayerShape(d=2048, E=16, f=512, k=4, f_shared=1024)])
def test_bad_expert_id_sets_device_error(ds4, shape):
    wl = synth.Workload("bad_id", shape, (1,), 0.0, 13)
    D = ds4.DeviceLayer(synth.make_layer(wl))
    x = dev(synth.activations(wl, 1)).view(torch.bfloat16)
    bad = [1, 99] + list(range(2, shape.k))  # 99 >= E: skipped on the device, flagged
    ids = torch.tensor([bad], dtype=torch.int32, device="cuda")
    w = torch.full((1, shape.k), 1.0 / shape.k, dtype=torch.float32, device="cuda")
    ds4.expert_ffn_decode(D.ex, x, ids, w, D.ws)
    assert ds4.last_device_error() == 6
    assert ds4.last_device_error() == 0  # read clears


def test_decode_graph_matches_eager(ds4):
    """The graph-replayed single-token decode runs the same launches as DeviceLayer.forward: bit-identical."""
    wl = synth.WORKLOADS["tiny"]
    L = synth.make_layer(wl)
    D = ds4.DeviceLayer(L, max_tokens=1)
    x = dev(synth.activations(wl, 4, stream=11))
    G = D.decode_graph()
    D.reserve(64)  # growing the layer's own buffers must not disturb the graph
    for t in range(4):
        want = D.forward(x[t:t + 1].view(torch.bfloat16)).clone()
        got = G(x[t:t + 1]).clone()
        torch.cuda.synchronize()
        assert ds4.last_device_error() == 0
        assert torch.equal(got, want), t


def test_decode_graph_with_host_buffers(ds4):
    """The graph that also holds the H2D copy of x and the D2H copy of the output gives the same bits as the
    eager decode, read from its pinned host output buffer after a synchronization."""
    wl = synth.WORKLOADS["tiny"]
    L = synth.make_layer(wl)
    D = ds4.DeviceLayer(L, max_tokens=1)
    xh = torch.from_numpy(synth.activations(wl, 4, stream=12)).pin_memory()
    G = D.decode_graph(host_io=True)
    assert G.out_host.device.type == "cpu" and G.out_host.is_pinned()
    for t in range(4):
        want = D.forward(xh[t:t + 1].cuda().view(torch.bfloat16)).cpu()
        got = G(xh[t:t + 1])
        torch.cuda.synchronize()
        assert ds4.last_device_error() == 0
        assert torch.equal(got, want), t
