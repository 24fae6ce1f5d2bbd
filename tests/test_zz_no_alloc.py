"""The allocation-free decode entry point (ds4moe_expert_ffn_decode_noalloc).

It exists for callers that cannot allocate device memory (an engine whose
memory planner owns all of HBM, a plugin host without an allocator): instead
of a caller workspace it uses a fixed 1 MiB scratch array compiled into the
library.  Through the C ABI, two calls in a row must match the regular
workspace entry point within the layer tolerance, and a layer too large for
the fixed scratch must be refused.  Collected last on purpose.
"""
import ctypes

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


@pytest.mark.parametrize("shape", [synth.WORKLOADS["tiny"].shape,
                                   synth.LayerShape(d=1024, E=16, f=512, k=4, f_shared=512)])
def test_noalloc_matches_workspace_entry_two_calls(ds4, shape):
    L = synth.make_layer(synth.Workload("noalloc", shape, (1,), 1.0, 31))
    D = ds4.DeviceLayer(L, max_tokens=1)
    x = synth.f32_to_bf16_bits(synth.rng(9, shape.d).normal(size=(2, shape.d)).astype(np.float32))
    for t in range(2):  # two calls in a row share (and overwrite) the same fixed scratch
        xt = torch.from_numpy(x[t:t + 1]).cuda().view(torch.bfloat16)
        ids, w = D.route(xt)
        ref = ds4.expert_ffn_decode(D.ex, xt, ids, w, D.ws)
        got = ds4.expert_ffn_decode_noalloc(D.ex, xt, ids, w)
        torch.cuda.synchronize()
        assert ds4.last_device_error() == 0
        parity.assert_output_close(got.double().cpu().numpy(), ref.double().cpu().numpy(), "noalloc call %d" % t)


def test_noalloc_rejects_layer_beyond_its_limits(ds4):
    # f_shared = 65536: the down kernel cannot stage the shared expert's h on chip, so the GEMV path (the only
    # one the fixed scratch serves) does not take the layer; refused before any launch
    ex = ds4.Experts(4096, 2048, 256, 65536, 0, 0, 1, 1 << 20, 1 << 21, 1 << 22, 1 << 24, 1 << 24, 1 << 24, 1 << 23,
                     1 << 25, 1 << 26, 1 << 27)
    fake = ctypes.c_void_p(1 << 20)
    rc = ds4.lib().ds4moe_expert_ffn_decode_noalloc(ctypes.byref(ex), fake, fake, fake, 8, fake, None)
    assert rc == 2  # DS4MOE_EUNSUPPORTED
