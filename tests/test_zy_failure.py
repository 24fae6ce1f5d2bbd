"""Device failure path: a bounded wait that runs out records DS4MOE_ETIMEOUT, and the context stays usable.

The self-test kernel waits (through the tensor-core kernels' bounded mbarrier wait) on a barrier nothing
arrives at; after the 2 s bound it sets the device error word.  Nothing traps, faults or hangs: the host
reads the status, and a decode afterwards still matches the eager path.
"""
import pytest

torch = pytest.importorskip("torch")

from bit_quantized_moe_02_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ds4():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_moe_02_b200 import ds4moe
    ds4moe.lib()
    return ds4moe


def test_bounded_wait_times_out_and_context_survives(ds4):
    assert ds4.last_device_error() == 0
    assert ds4.lib().ds4moe_selftest_wait_timeout(ds4._stream()) == 0
    assert ds4.last_device_error() == 5  # DS4MOE_ETIMEOUT, read and cleared
    assert ds4.last_device_error() == 0
    wl = synth.WORKLOADS["tiny"]
    D = ds4.DeviceLayer(synth.make_layer(wl), max_tokens=1)
    x = torch.from_numpy(synth.activations(wl, 1)).cuda().view(torch.bfloat16)
    a = D.forward(x).clone()
    b = D.forward(x).clone()
    torch.cuda.synchronize()
    assert ds4.last_device_error() == 0
    assert torch.isfinite(a).all() and torch.equal(a, b)
