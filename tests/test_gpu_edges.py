"""Degenerate and extreme cases of the layer, through the C ABI against the oracle.

- every token routed to the same k experts (router bias forcing the choice): k experts with T tokens each,
  so each expert spans several token tiles with a ragged last one, and every other expert is empty;
- a single token through the grouped and the fused prefill calls (one tile of one token, padded to 16);
- k = E (every expert selected);
- E = 1024, the grouped path's largest expert count (one CTA scans all expert counts);
- f = 16384, the grouped path's longest down contraction (one h scale per 128-wide K range held on chip), which
  the single-token GEMV does not take, so B = 1 decode runs the grouped path too.
Each case runs the deterministic grouped call, the fused call and single-token decode, compared with the oracle
at the layer tolerance.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

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


def tokens(seed, T, d):
    return synth.f32_to_bf16_bits(synth.rng(seed, T, d).normal(size=(T, d)).astype(np.float32))


def run(ds4, L, x, paths=("grouped", "fused", "decode"), n_decode=2):
    D = ds4.DeviceLayer(L, max_tokens=x.shape[0])
    xt = torch.from_numpy(x).cuda().view(torch.bfloat16)
    ref = parity.oracle_layer(L, x)
    for path in paths:
        if path == "grouped":
            out, ids, _, _, _ = D.forward_grouped(xt)
            rows = np.arange(x.shape[0])
        elif path == "fused":
            out, ids, _ = D.forward_fused(xt)
            rows = np.arange(x.shape[0])
        else:
            outs, idss = [], []
            for t in range(n_decode):
                o, i, _ = D.forward(xt[t:t + 1], return_routing=True)
                outs.append(o)
                idss.append(i)
            out, ids = torch.cat(outs), torch.cat(idss)
            rows = np.arange(n_decode)
        torch.cuda.synchronize()
        assert ds4.last_device_error() == 0, path
        sub = {key: (v[rows] if isinstance(v, np.ndarray) and v.shape[:1] == (x.shape[0],) else v)
               for key, v in ref.items()}
        want, _ = parity.check_ids(ids.cpu().numpy(), sub)
        got = out.double().cpu().numpy()
        assert np.all(np.isfinite(got)), path
        parity.assert_output_close(got, want, path)


@pytest.mark.parametrize("T", [300, 129])
def test_every_token_on_the_same_experts(ds4, T):
    shape = synth.LayerShape(d=512, E=16, f=512, k=4, f_shared=256)
    L = synth.make_layer(synth.Workload("edges", shape, (1,), 0.0, 90 + T))
    L.bias = np.zeros(shape.E, np.float32)
    L.bias[[3, 7, 11, 12]] = [10.0, 9.0, 8.0, 7.0]  # far above any logit: these four win for every token
    x = tokens(91, T, shape.d)
    ref = parity.oracle_layer(L, x[:4])
    assert all(sorted(r) == [3, 7, 11, 12] for r in ref["ids"].tolist())
    run(ds4, L, x)


def test_single_token_grouped_and_fused(ds4):
    wl = synth.WORKLOADS["tiny"]
    L = synth.make_layer(wl)
    run(ds4, L, synth.activations(wl, 1), n_decode=1)


def test_every_expert_selected(ds4):
    shape = synth.LayerShape(d=256, E=8, f=256, k=8, f_shared=256)
    L = synth.make_layer(synth.Workload("edges", shape, (1,), 1.0, 92))
    run(ds4, L, tokens(93, 40, shape.d))


def test_thousand_experts(ds4):
    shape = synth.LayerShape(d=256, E=1024, f=256, k=2, f_shared=0)
    L = synth.make_layer(synth.Workload("edges", shape, (1,), 1.0, 94))
    run(ds4, L, tokens(95, 200, shape.d))


def test_longest_down_contraction(ds4):
    shape = synth.LayerShape(d=256, E=4, f=16384, k=2, f_shared=256)
    L = synth.make_layer(synth.Workload("edges", shape, (1,), 1.0, 96))
    run(ds4, L, tokens(97, 40, shape.d))
