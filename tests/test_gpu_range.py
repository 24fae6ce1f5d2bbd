"""Range of the fp16 intermediates, on adversarial but legal inputs, through the C ABI against the oracle.

The decode GEMV multiplies fp16 pairs and adds them in fp16 inside each 32-weight IQ2X group (activations scaled
so that max |x| lies in [32, 64); a codebook value is at most 43) and inside each 16-weight Q2K sub-block (staged
h scaled the same way; q <= 3).  Each fp16 lane of a group sum then holds 16 products, at most
16 * 43 * 64 = 44,032 < 65,504, and a sub-block lane 4 products of at most 3 * 64: no overflow is possible for
finite inputs.  These tests drive those sums to their bounds (a codebook row of all 43, all signs positive, the
largest group scale s = 15, every activation at the token's maximum; Q2K with sc = 15 and q = 3 everywhere) and
compare with the oracle at the layer tolerance.  The grouped (prefill) path stores the SwiGLU output h in fp16 with
a power-of-two scale per token tile and 128-row block; a layer whose h exceeds 65,504 must still match the oracle.
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


def f16(v):
    return int(np.float16(v).view(np.uint16))


def iq2x_const(rows, cols, d, s=15):
    """Every 8-vector: codebook entry 0, no negative sign, group scale s, block scale d."""
    blk = np.zeros(66, np.uint8)
    blk[0], blk[1] = f16(d) & 0xFF, f16(d) >> 8
    for g in range(8):
        aux = s << 28
        blk[2 + 8 * g + 4:2 + 8 * g + 8] = np.frombuffer(np.uint32(aux).tobytes(), np.uint8)
    return np.tile(blk, rows * (cols // 256)).reshape(rows, -1)


def q2k_const(rows, cols, d, dmin, sc=15, m=0, q=3):
    """Every sub-block: scale sc, min m, every code q."""
    blk = np.zeros(84, np.uint8)
    blk[:16] = sc | (m << 4)
    blk[16:80] = q | (q << 2) | (q << 4) | (q << 6)
    blk[80], blk[81] = f16(d) & 0xFF, f16(d) >> 8
    blk[82], blk[83] = f16(dmin) & 0xFF, f16(dmin) >> 8
    return np.tile(blk, rows * (cols // 256)).reshape(rows, -1)


def fixed_layer(shape, seed, gate=None, up=None, down=None, grid_row0=None, bias_std=0.0):
    """A seeded layer whose expert matrices are replaced by the given canonical arrays (same for every expert)."""
    L = synth.make_layer(synth.Workload("range", shape, (1,), bias_std, seed))
    fixed = {"gate": gate, "up": up, "down": down}
    rand = L.expert

    def expert(which, e):
        return fixed[which] if fixed[which] is not None else rand(which, e)

    L.expert = expert
    L.drop_cache = lambda: None
    if grid_row0 is not None:
        L.grid = L.grid.copy()
        L.grid[0] = grid_row0
    return L


def compare(ds4, L, x, path):
    D = ds4.DeviceLayer(L, max_tokens=x.shape[0])
    xt = torch.from_numpy(x).cuda().view(torch.bfloat16)
    if path == "decode":
        outs, idss = [], []
        for t in range(x.shape[0]):
            o, ids, _ = D.forward(xt[t:t + 1], return_routing=True)
            outs.append(o)
            idss.append(ids)
        out, ids = torch.cat(outs), torch.cat(idss)
    elif path == "fused":
        out, ids, _ = D.forward_fused(xt)
    else:
        out, ids, _, _, _ = D.forward_grouped(xt)
    torch.cuda.synchronize()
    assert ds4.last_device_error() == 0
    ref = parity.oracle_layer(L, x)
    want, _ = parity.check_ids(ids.cpu().numpy(), ref)
    got = out.double().cpu().numpy()
    assert np.all(np.isfinite(got))
    return parity.assert_output_close(got, want, path)


# the token's activations all at their maximum: 1.9921875 (bf16 0x3FFF) scales to 63.75, the top of [32, 64)
X_MAX = np.uint16(0x3FFF)


@pytest.mark.parametrize("d", [4096, 2048, 768])
def test_decode_group_sums_at_their_bound(ds4, d):
    shape = synth.LayerShape(d=d, E=8, f=256, k=2, f_shared=256)
    g = iq2x_const(shape.f, d, 1e-3)
    L = fixed_layer(shape, 61, gate=g, up=g, grid_row0=np.full(8, 43, np.uint8))
    x = np.full((2, d), X_MAX, np.uint16)
    x[1, ::2] = np.uint16(0xBFFF)  # second token: alternating signs, same magnitude
    compare(ds4, L, x, "decode")


def test_decode_q2k_sub_blocks_at_their_bound(ds4):
    shape = synth.LayerShape(d=1024, E=8, f=2048, k=2, f_shared=512)
    g = iq2x_const(shape.f, shape.d, 1e-3)
    dn = q2k_const(shape.d, shape.f, 1e-3, 2e-4, sc=15, m=15, q=3)
    L = fixed_layer(shape, 62, gate=g, up=g, down=dn, grid_row0=np.full(8, 43, np.uint8))
    x = np.full((2, shape.d), X_MAX, np.uint16)
    compare(ds4, L, x, "decode")


@pytest.mark.parametrize("path", ["grouped", "fused"])
def test_grouped_swiglu_output_beyond_fp16(ds4, path):
    """Block scales d = 0.25 make |h| reach about 1e8 (far beyond fp16): the grouped path scales the stored h by a
    power of two per token tile and row block and the down GEMM multiplies the weights back."""
    shape = synth.LayerShape(d=512, E=8, f=512, k=2, f_shared=256)
    L = synth.make_layer(synth.Workload("range", shape, (1,), 1.0, 63))
    rand = L.expert

    def big(which, e):
        a = rand(which, e).copy()
        if which in ("gate", "up"):
            blocks = a.reshape(-1, 66)
            blocks[:, 0], blocks[:, 1] = f16(0.25) & 0xFF, f16(0.25) >> 8
        return a

    L.expert = big
    L.drop_cache = lambda: None
    x = synth.f32_to_bf16_bits(synth.rng(64).normal(0, 4.0, size=(150, shape.d)).astype(np.float32))
    rel, mx = compare(ds4, L, x, path)
    ref = parity.oracle_layer(L, x[:4])
    assert np.abs(ref["out"]).max() > 1e6  # the case really is beyond the fp16 range


@pytest.mark.parametrize("d,f,fs", [(768, 512, 256), (3072, 1024, 512), (1280, 768, 768)])
def test_decode_gemv_other_widths(ds4, d, f, fs):
    """B = 1 decode on layers whose d (and f) are not 256 times a power of two: outside the single-token GEMV
    kernels' shapes, so the call takes the grouped path with one token; checked against the oracle like any
    other layer."""
    shape = synth.LayerShape(d=d, E=16, f=f, k=4, f_shared=fs)
    L = synth.make_layer(synth.Workload("widths", shape, (1,), 1.0, 70 + d))
    x = synth.f32_to_bf16_bits(synth.rng(71, d).normal(size=(3, d)).astype(np.float32))
    compare(ds4, L, x, "decode")
