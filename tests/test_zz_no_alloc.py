"""The allocation-free decode entry point (ds4moe_expert_ffn_decode_noalloc).

It exists for callers that cannot allocate device memory (an engine whose
memory planner owns all of HBM, a plugin host without an allocator): instead
of a caller workspace it uses a fixed 1 MiB scratch array compiled into the
library.  Through the C ABI, two calls in a row must give exactly the output of
the regular workspace entry point (both run the same two kernels on the same
inputs), one of them is also checked against the oracle, and a layer beyond
the GEMV path's limits must be refused.  Collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from bit_quantized_moe_02_b200 import ds4moe as ds4binding
from bit_quantized_moe_02_b200 import synth
from tests import parity


@pytest.fixture(scope="module")
def ds4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ds4binding.lib()
    return ds4binding


# the decode layer's shape (d=4096, f=2048, k=8, shared 2048) with 16 experts: the scratch and the kernel variants
# depend on d, f, k and f_shared only, not on E
DECODE_SHAPE_E16 = synth.LayerShape(d=4096, E=16, f=2048, k=8, f_shared=2048)


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [synth.WORKLOADS["tiny"].shape,
                                   synth.LayerShape(d=1024, E=16, f=512, k=4, f_shared=512),
                                   DECODE_SHAPE_E16])
def test_noalloc_matches_workspace_entry_two_calls(ds4, shape):
    L = synth.make_layer(synth.Workload("noalloc", shape, (1,), 1.0, 31))
    D = ds4.DeviceLayer(L, max_tokens=1)
    x = synth.f32_to_bf16_bits(synth.rng(9, shape.d).normal(size=(2, shape.d)).astype(np.float32))
    for t in range(2):  # two calls in a row share (and overwrite) the same fixed scratch
        xt = torch.from_numpy(x[t:t + 1]).cuda().view(torch.bfloat16)
        ids, w = D.route(xt)
        ref = ds4.expert_ffn_decode(D.ex, xt, ids, w, D.ws).clone()
        got = ds4.expert_ffn_decode_noalloc(D.ex, xt, ids, w).clone()
        torch.cuda.synchronize()
        assert ds4.last_device_error() == 0
        assert torch.equal(got, ref), "noalloc call %d differs from the workspace entry point" % t
        if t == 1:  # and independently against the oracle
            want, _ = parity.check_ids(ids.cpu().numpy(), parity.oracle_layer(L, x[t:t + 1]))
            parity.assert_output_close(got.double().cpu().numpy(), want, "noalloc vs oracle")


@pytest.mark.gpu
def test_noalloc_rejects_layer_beyond_its_limits(ds4):
    # d = 3072 (not 256 times a power of two): outside the GEMV path, the only one the fixed scratch serves;
    # refused before any launch
    ex = ds4.Experts(3072, 2048, 256, 2048, 0, 0, 1, 1 << 20, 1 << 21, 1 << 22, 1 << 24, 1 << 24, 1 << 24, 1 << 23,
                     1 << 25, 1 << 26, 1 << 27)
    fake = ctypes.c_void_p(1 << 20)
    rc = ds4.lib().ds4moe_expert_ffn_decode_noalloc(ctypes.byref(ex), fake, fake, fake, 8, fake, None)
    assert rc == 2  # DS4MOE_EUNSUPPORTED


@pytest.mark.skipif(torch.cuda.is_available(), reason="calls with stand-in pointers would launch on a GPU")
def test_every_gemv_layer_fits_the_fixed_scratch():
    """No GPU: for every layer shape the single-token GEMV path accepts (probed through ds4moe_decode_gateup, which
    refuses the others with DS4MOE_EUNSUPPORTED before any launch), the allocation-free call gets past its scratch
    size check (DS4MOE_ENOWORKSPACE would mean the 1 MiB array is too small) and stops only at the device lookup."""
    lib = ds4binding.lib()
    fake = ctypes.c_void_p(1 << 20)
    accepted = 0
    for d in (256, 1024, 2048, 4096, 8192):
        for f in (256, 1024, 2048, 4096, 8192):
            for fs in (0, 2048, 4096):
                for k in (1, 8, 16, 32):
                    ex = ds4binding.Experts(d, f, 64, fs, 0, 0, 1, 1 << 20, 1 << 21, 1 << 22, 1 << 26, 1 << 26,
                                            1 << 26, 1 << 23, 1 << 24 if fs else None, 1 << 25 if fs else None,
                                            1 << 27 if fs else None)
                    if lib.ds4moe_decode_gateup(ctypes.byref(ex), fake, fake, k, fake, 1 << 30, None) == 2:
                        continue  # not a GEMV layer
                    accepted += 1
                    rc = lib.ds4moe_expert_ffn_decode_noalloc(ctypes.byref(ex), fake, fake, fake, k, fake, None)
                    assert rc not in (2, 4), (d, f, fs, k, rc)
    assert accepted > 50
