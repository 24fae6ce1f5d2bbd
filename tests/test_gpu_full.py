"""Full-size workloads through the C ABI against the oracle on seeded token subsets.

prefill: the decode-sized layer (d=4096, E=256, f=2048, k=8, shared 2048) at
T=4096 with skewed routing, compared on 256 sampled tokens; q4: the same layer
with Q4K experts at T=16384, then one decode token.  The layer is per-token
independent, so the oracle on a subset is exact.
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


def compare_subset(ds4, L, x, out, ids, sample):
    ref = parity.oracle_layer(L, x[sample])
    want, _ = parity.check_ids(ids.cpu().numpy()[sample], ref)
    gpu = out.double().cpu().numpy()[sample]
    return parity.assert_output_close(gpu, want)


@pytest.mark.parametrize("name", ["prefill", "q4"])
def test_full_prefill(ds4, name):
    wl = synth.WORKLOADS[name]
    T = wl.tokens[0]
    L = synth.make_layer(wl)
    x = synth.activations(wl, T)
    D = ds4.DeviceLayer(L, max_tokens=T)
    xt = torch.from_numpy(x).cuda().view(torch.bfloat16)
    out, ids, w, y_perm, inv = D.forward_grouped(xt)
    torch.cuda.synchronize()
    assert ds4.last_device_error() == 0
    # every (token, slot) pair lands exactly once, and within an expert in (token, slot) order
    inv_np = inv.cpu().numpy()
    assert np.array_equal(np.sort(inv_np), np.arange(T * wl.shape.k))
    ids_np = ids.cpu().numpy().reshape(-1)
    order = np.argsort(inv_np)
    assert np.all(np.diff(ids_np[order]) >= 0)
    sample = synth.sample_tokens(wl, T, 256)
    compare_subset(ds4, L, x, out, ids, sample)
    # the deterministic path is bit-reproducible: a second call on the same input gives identical rows (this
    # catches a pipeline race in the grouped kernels, which shows as a few stale weight rows in some tiles)
    out2, ids2, _, y_perm2, _ = D.forward_grouped(xt)
    torch.cuda.synchronize()
    assert torch.equal(ids2, ids) and torch.equal(y_perm2, y_perm) and torch.equal(out2, out)
    del out2, y_perm2
    # the fused-combine call on the same tokens: same routing, same output up to fp32 summation order
    fused, ids_f, _ = D.forward_fused(xt)
    torch.cuda.synchronize()
    assert ds4.last_device_error() == 0
    assert torch.equal(ids_f, ids)
    assert float((fused - out).abs().max()) <= 1e-5 * float(out.abs().max())
    compare_subset(ds4, L, x, fused, ids, sample)
    if name == "q4":
        x1 = synth.activations(wl, 1, stream=1)
        o1, ids1, _ = D.forward(torch.from_numpy(x1).cuda().view(torch.bfloat16), return_routing=True)
        torch.cuda.synchronize()
        compare_subset(ds4, L, x1, o1, ids1, np.arange(1))
