"""The binding's tensor checks (no GPU): every call pattern the package, tests and benchmark use passes them, and a
host tensor, a wrong shape or element size, a non-contiguous or a short buffer raises before the library is
called.  CUDA tensors are stood in for by objects with the same attributes; the library by a recorder."""
import types

import pytest

torch = pytest.importorskip("torch")

from bit_quantized_moe_02_b200 import ds4moe  # noqa: E402


class FakeCuda:
    def __init__(self, shape, dtype, dev=0, contiguous=True):
        self._t = torch.empty(shape, dtype=dtype)
        self.shape = self._t.shape
        self.dtype = dtype
        self.is_cuda = True
        self.device = types.SimpleNamespace(index=dev, type="cuda")
        self._contiguous = contiguous

    def is_contiguous(self):
        return self._contiguous

    def element_size(self):
        return self._t.element_size()

    def numel(self):
        return self._t.numel()

    def data_ptr(self):
        return 1 << 20


class Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append(name)
            return 4096 if name.endswith(("_size", "_bytes")) else 0
        return fn


@pytest.fixture
def rec(monkeypatch):
    r = Recorder()
    monkeypatch.setattr(ds4moe, "lib", lambda: r)
    monkeypatch.setattr(ds4moe, "_cur", lambda: 0)
    monkeypatch.setattr(ds4moe, "_stream", lambda: None)
    return r


D, F, E, K, T = 512, 256, 16, 4, 7
bf16, f16, f32, i32, u8 = torch.bfloat16, torch.float16, torch.float32, torch.int32, torch.uint8


def experts():
    return ds4moe.Experts(D, F, E, F, 0, 0, 1)


def test_call_patterns_in_use_pass(rec):
    ex = experts()
    ws = FakeCuda((4096,), u8)
    # single-token decode, as DeviceLayer.forward, DecodeGraph and the benchmark issue it
    x1, ids1, w1, out1 = FakeCuda((1, D), bf16), FakeCuda((1, K), i32), FakeCuda((1, K), f32), FakeCuda((1, D), f32)
    ds4moe.route(x1, FakeCuda((E, D), f16), FakeCuda((E,), f32), K, ws=ws, ids=ids1, weights=w1)
    ds4moe.route(FakeCuda((T, D), torch.uint16), FakeCuda((E, D), f16), None, K, ws=ws,
                 ids=FakeCuda((T, K), i32), weights=FakeCuda((T, K), f32))  # bf16 bits as uint16
    ds4moe.expert_ffn_decode(ex, x1, ids1, w1, ws, out=out1)
    ds4moe.decode_gateup(ex, x1, ids1, ws)
    ds4moe.decode_down(ex, ids1, w1, ws, out1)
    ds4moe.expert_ffn_decode_noalloc(ex, x1, ids1, w1, out=out1)
    # many tokens: grouped experts and combine, with and without a shared expert output
    xT, idsT, wT = FakeCuda((T, D), bf16), FakeCuda((T, K), i32), FakeCuda((T, K), f32)
    y_perm, inv, ys = FakeCuda((T * K, D), f32), FakeCuda((T * K,), i32), FakeCuda((T, D), f32)
    ds4moe.expert_ffn_decode(ex, xT, idsT, wT, ws, out=FakeCuda((T, D), f32))
    for y_sh in (ys, None):
        ds4moe.expert_ffn_grouped(ex, xT, idsT, wT, ws, y_perm, inv, y_sh)
        ds4moe.combine(y_perm, inv, y_sh, T, D, K, out=FakeCuda((T, D), f32))
    # repack: a chunk of canonical matrices into a slice of the layer's buffer
    stride = 4096  # the recorder's prepared size, already a multiple of 256
    ds4moe.prepare("q2k", FakeCuda((3, D * F // 256 * 84), u8), D, F, 3, out=FakeCuda((stride * 5,), u8))
    with pytest.raises(ValueError):  # the chunk does not fit in what is left of the buffer
        ds4moe.prepare("q2k", FakeCuda((3, D * F // 256 * 84), u8), D, F, 3, out=FakeCuda((stride * 2,), u8))
    assert rec.calls.count("ds4moe_route") == 2 and rec.calls.count("ds4moe_prepare") == 1
    assert rec.calls.count("ds4moe_expert_ffn_grouped") == 2 and rec.calls.count("ds4moe_combine") == 2


@pytest.mark.parametrize("case", ["host", "other_device", "shape", "esize", "contiguous", "short"])
def test_bad_arguments_raise_before_the_library(rec, case):
    ex = experts()
    ws = FakeCuda((4096,), u8)
    x, ids, w, out = FakeCuda((1, D), bf16), FakeCuda((1, K), i32), FakeCuda((1, K), f32), FakeCuda((1, D), f32)
    inv = FakeCuda((T * K,), i32)
    with pytest.raises(ValueError):
        if case == "host":
            ds4moe.expert_ffn_decode(ex, torch.zeros((1, D), dtype=bf16), ids, w, ws, out=out)
        elif case == "other_device":
            ds4moe.expert_ffn_decode(ex, FakeCuda((1, D), bf16, dev=1), ids, w, ws, out=out)
        elif case == "shape":
            ds4moe.route(x, FakeCuda((E, D), f16), None, K, ws=ws, ids=FakeCuda((2, K), i32), weights=w)
        elif case == "esize":
            ds4moe.expert_ffn_decode(ex, FakeCuda((1, D), f32), ids, w, ws, out=out)
        elif case == "contiguous":
            ds4moe.decode_down(ex, ids, w, ws, FakeCuda((1, D), f32, contiguous=False))
        else:
            ds4moe.combine(FakeCuda((T * K - 1, D), f32), inv, None, T, D, K, out=FakeCuda((T, D), f32))
    assert not any(c.startswith("ds4moe_") and not c.endswith(("_size", "_bytes")) for c in rec.calls)
