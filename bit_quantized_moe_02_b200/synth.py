"""Seeded synthetic inputs for the 2-bit routed-MoE FFN layer.

This module only draws random numbers and packs them into the byte layouts the
layer consumes; it performs none of the layer's arithmetic (no dequantization,
no routing, no contraction).  Both the CPU oracle (through the tests) and the
CUDA path consume exactly these arrays, so it is the one module the two sides
share.

Workloads (sizes from the ds4 pages' model description: routed experts
quantized, shared expert / router left in high precision -- ds4 news summary,
"model weights" section; upppp.jp article, "asymmetric 2-bit quantization"):

  tiny      d=256,  E=8,   f=512,  k=2, shared f=512,  1 token, no bias
  decode    d=4096, E=256, f=2048, k=8, shared f=2048, 1 token, no bias
  batched   the decode layer at B in {1,4,16,64}, router bias N(0,1)
  prefill   the decode layer at T=4096, router bias N(0,1)
  q4        the decode layer with Q4K-style experts, T=16384 then B=1

Every tensor is drawn from numpy PCG64 seeded by SeedSequence([seed, layer,
tag, index]) so any single expert can be regenerated on its own.

Byte layouts written here (little endian; see include/ds4moe.h):
  IQ2X block, 66 B / 256 weights: fp16 d at bytes 0..1, then 8 groups of
      idx[4] u8 + aux u32 (aux: 4 x 7 sign bits, 4-bit scale in bits 28..31).
  Q2K block, 84 B / 256 weights: scales[16] (sc | m<<4), qs[64], fp16 d, fp16 dmin.
  Q4K block, 144 B / 256 weights: fp16 d, fp16 dmin, 12 scale bytes, qs[128].
Quant bytes are uniform random; d and dmin are |N(0, 1e-3)| rounded to fp16.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np

QK = 256
FMTS = ("iq2x", "q2k", "q4k")
BLOCK_BYTES = {"iq2x": 66, "q2k": 84, "q4k": 144}
# byte offsets of the fp16 super-block scales inside one block
_D_OFFSETS = {"iq2x": (0,), "q2k": (80, 82), "q4k": (0, 2)}
GRID_VALUES = (8, 25, 43)

TAG_X, TAG_WR, TAG_BIAS, TAG_GRID = 1, 2, 3, 4
TAG_GATE, TAG_UP, TAG_DOWN = 5, 6, 7
TAG_SH_GATE, TAG_SH_UP, TAG_SH_DOWN = 8, 9, 10
TAG_SAMPLE = 11


def rng(*tags: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(t) for t in tags])))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest-even) and return the raw uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    return ((u + rounding) >> 16).astype(np.uint16)


def f32_to_f16_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


@dataclasses.dataclass(frozen=True)
class LayerShape:
    d: int
    E: int
    f: int
    k: int
    f_shared: int
    fmt_gate: str = "iq2x"
    fmt_up: str = "iq2x"
    fmt_down: str = "q2k"

    def mat_bytes(self, fmt: str, rows: int, cols: int) -> int:
        return rows * (cols // QK) * BLOCK_BYTES[fmt]

    @property
    def expert_bytes(self) -> int:
        return (self.mat_bytes(self.fmt_gate, self.f, self.d) + self.mat_bytes(self.fmt_up, self.f, self.d)
                + self.mat_bytes(self.fmt_down, self.d, self.f))

    @property
    def shared_bytes(self) -> int:
        return 2 * 3 * self.f_shared * self.d

    @property
    def router_bytes(self) -> int:
        return 2 * self.E * self.d


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: LayerShape
    tokens: Sequence[int]
    bias_std: float
    seed: int


_DECODE = LayerShape(d=4096, E=256, f=2048, k=8, f_shared=2048)
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", LayerShape(d=256, E=8, f=512, k=2, f_shared=512), (1,), 0.0, 0),
    "decode": Workload("decode", _DECODE, (1,), 0.0, 1),
    "batched": Workload("batched", _DECODE, (1, 4, 16, 64), 1.0, 2),
    "prefill": Workload("prefill", _DECODE, (4096,), 1.0, 3),
    "q4": Workload("q4", dataclasses.replace(_DECODE, fmt_gate="q4k", fmt_up="q4k", fmt_down="q4k"),
                   (16384, 1), 1.0, 4),
}


def random_blocks(fmt: str, n_blocks: int, g: np.random.Generator) -> np.ndarray:
    """n_blocks canonical blocks of `fmt` as a uint8 array [n_blocks, block_bytes]."""
    bb = BLOCK_BYTES[fmt]
    raw = np.frombuffer(g.bytes(n_blocks * bb), dtype=np.uint8).reshape(n_blocks, bb).copy()
    for off in _D_OFFSETS[fmt]:
        dv = f32_to_f16_bits(np.abs(g.normal(0.0, 1e-3, size=n_blocks)).astype(np.float32))
        raw[:, off] = (dv & 0xFF).astype(np.uint8)
        raw[:, off + 1] = (dv >> 8).astype(np.uint8)
    return raw


def random_matrix(fmt: str, rows: int, cols: int, g: np.random.Generator) -> np.ndarray:
    """Canonical quantized matrix [rows, cols/256 * block_bytes] (blocks run along cols)."""
    assert cols % QK == 0
    nb = cols // QK
    return random_blocks(fmt, rows * nb, g).reshape(rows, nb * BLOCK_BYTES[fmt])


def codebook(seed: int) -> np.ndarray:
    """256 x 8 uint8 grid of values drawn uniformly from {8, 25, 43}."""
    g = rng(seed, 0, TAG_GRID)
    return np.asarray(GRID_VALUES, dtype=np.uint8)[g.integers(0, 3, size=(256, 8))]


@dataclasses.dataclass
class Layer:
    """Host copy of one layer's inputs.  Expert matrices are generated lazily per expert."""
    wl: Workload
    layer: int
    wr: np.ndarray            # uint16 fp16 bits [E, d]
    bias: np.ndarray          # float32 [E]
    grid: np.ndarray          # uint8 [256, 8]
    sh_gate: Optional[np.ndarray]  # uint16 bf16 bits [f_s, d]
    sh_up: Optional[np.ndarray]
    sh_down: Optional[np.ndarray]  # [d, f_s]
    _cache: Dict = dataclasses.field(default_factory=dict)

    @property
    def shape(self) -> LayerShape:
        return self.wl.shape

    def expert(self, which: str, e: int) -> np.ndarray:
        key = (which, e)
        if key not in self._cache:
            s = self.shape
            tag, fmt, rows, cols = {
                "gate": (TAG_GATE, s.fmt_gate, s.f, s.d),
                "up": (TAG_UP, s.fmt_up, s.f, s.d),
                "down": (TAG_DOWN, s.fmt_down, s.d, s.f),
            }[which]
            self._cache[key] = random_matrix(fmt, rows, cols, rng(self.wl.seed, self.layer, tag, e))
        return self._cache[key]

    def all_experts(self, which: str) -> np.ndarray:
        """All E matrices stacked: [E, rows, row_bytes] (generated once, then cached)."""
        return np.stack([self.expert(which, e) for e in range(self.shape.E)])

    def drop_cache(self) -> None:
        self._cache.clear()


def make_layer(wl: Workload, layer: int = 0) -> Layer:
    s = wl.shape
    seed = wl.seed
    wr = f32_to_f16_bits(rng(seed, layer, TAG_WR).normal(0.0, 0.02, size=(s.E, s.d)).astype(np.float32))
    if wl.bias_std > 0:
        bias = rng(seed, layer, TAG_BIAS).normal(0.0, wl.bias_std, size=s.E).astype(np.float32)
    else:
        bias = np.zeros(s.E, dtype=np.float32)
    sh = [None, None, None]
    if s.f_shared > 0:
        for i, (tag, shp) in enumerate(((TAG_SH_GATE, (s.f_shared, s.d)), (TAG_SH_UP, (s.f_shared, s.d)),
                                        (TAG_SH_DOWN, (s.d, s.f_shared)))):
            sh[i] = f32_to_bf16_bits(rng(seed, layer, tag).normal(0.0, 0.02, size=shp).astype(np.float32))
    return Layer(wl, layer, wr, bias, codebook(seed), sh[0], sh[1], sh[2])


def activations(wl: Workload, T: int, layer: int = 0, stream: int = 0) -> np.ndarray:
    """x: uint16 bf16 bits [T, d], N(0, 1)."""
    g = rng(wl.seed, layer, TAG_X, T, stream)
    return f32_to_bf16_bits(g.normal(0.0, 1.0, size=(T, wl.shape.d)).astype(np.float32))


def sample_tokens(wl: Workload, T: int, n: int) -> np.ndarray:
    """Seeded subset of token indices compared against the oracle at large T."""
    if n >= T:
        return np.arange(T)
    return np.sort(rng(wl.seed + 1000, TAG_SAMPLE, T).choice(T, size=n, replace=False))
