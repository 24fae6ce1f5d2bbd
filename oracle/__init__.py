"""CPU oracle for the 2-bit routed-MoE FFN -- test infrastructure only.

Thin ctypes front end over ``ds4moe_oracle.c`` (plain C, fp32 dequantization
in the block definitions' op order, fp64 contraction).  Only the tests, the
package's smoke check and the benchmark's CPU-baseline leg may import this
package; the product path never does.  It imports nothing from the CUDA
library and the CUDA library imports nothing from it.

Everything takes plain numpy arrays: canonical block bytes (uint8), raw fp16 /
bf16 bit patterns (uint16) and float32 router biases.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Callable, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ds4moe_oracle.c")
_LIB = os.path.join(_HERE, "libds4moe_oracle.so")
FMT_CODE = {"iq2x": 0, "q2k": 1, "q4k": 2}
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                               "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Layer(ctypes.Structure):
    _fields_ = [
        ("d", ctypes.c_int), ("f", ctypes.c_int), ("E", ctypes.c_int), ("k", ctypes.c_int),
        ("f_shared", ctypes.c_int),
        ("fmt_gate", ctypes.c_int), ("fmt_up", ctypes.c_int), ("fmt_down", ctypes.c_int),
        ("gate", ctypes.POINTER(ctypes.c_void_p)), ("up", ctypes.POINTER(ctypes.c_void_p)),
        ("down", ctypes.POINTER(ctypes.c_void_p)),
        ("grid", ctypes.c_void_p),
        ("sh_gate", ctypes.c_void_p), ("sh_up", ctypes.c_void_p), ("sh_down", ctypes.c_void_p),
        ("wr", ctypes.c_void_p), ("bias", ctypes.c_void_p),
    ]


def lib():
    global _lib
    if _lib is None:
        # DS4MOE_ORACLE_LIB lets the pin tests load a deliberately broken copy of the oracle
        l = ctypes.CDLL(os.environ.get("DS4MOE_ORACLE_LIB") or build())
        l.orc_dequant.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
        l.orc_route.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                ctypes.c_void_p, ctypes.c_void_p]
        l.orc_layer_forward.argtypes = [ctypes.POINTER(_Layer), ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p]
        _lib = l
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def dequant(fmt: str, blocks: np.ndarray, grid: Optional[np.ndarray] = None) -> np.ndarray:
    """Canonical blocks (uint8, any shape whose size is a multiple of the block size) -> float32 weights."""
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    bb = {"iq2x": 66, "q2k": 84, "q4k": 144}[fmt]
    assert blocks.size % bb == 0
    nb = blocks.size // bb
    out = np.empty(nb * 256, dtype=np.float32)
    g = None if grid is None else np.ascontiguousarray(grid, dtype=np.uint8)
    rc = lib().orc_dequant(FMT_CODE[fmt], _ptr(blocks), nb, _ptr(g), _ptr(out))
    if rc != 0:
        raise ValueError("oracle dequant rejected its arguments")
    return out


def route(x: np.ndarray, wr: np.ndarray, bias: Optional[np.ndarray], k: int, alt: bool = False):
    """Sigmoid router + top-k.  Returns ids [T,k] int32, w [T,k] f64, scores [T,E] f64, gap [T] f64."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    wr = np.ascontiguousarray(wr, dtype=np.uint16)
    T, d = x.shape
    E = wr.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    scores = np.empty((T, E), np.float64)
    gap = np.empty(T, np.float64)
    rc = lib().orc_route(_ptr(x), T, d, _ptr(wr), _ptr(b), E, k, int(alt), _ptr(ids), _ptr(w), _ptr(scores),
                         _ptr(gap))
    if rc != 0:
        raise ValueError("oracle route rejected its arguments")
    return ids, w, scores, gap


def layer_forward(shape, x: np.ndarray, wr: np.ndarray, bias: Optional[np.ndarray], grid: np.ndarray,
                  expert: Callable[[str, int], np.ndarray], shared: Sequence[Optional[np.ndarray]],
                  alt: bool = False, nthreads: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray, np.ndarray,
                                                                             np.ndarray]:
    """Whole MoE FFN layer for tokens x [T, d] (bf16 bits).

    ``shape`` has d, E, f, k, f_shared, fmt_gate, fmt_up, fmt_down.  ``expert(which, e)`` returns the
    canonical matrix of expert e ('gate' / 'up' [f x d], 'down' [d x f]); it is only called for the experts
    the tokens select.  Returns out [T, d] f64, ids [T, k], w [T, k], gap [T].
    """
    x = np.ascontiguousarray(x, dtype=np.uint16)
    T = x.shape[0]
    k, E = shape.k, shape.E
    ids0, _, _, _ = route(x, wr, bias, k, alt=False)
    need = set(int(e) for e in ids0.ravel())
    if alt:
        ids1, _, _, _ = route(x, wr, bias, k, alt=True)
        need |= set(int(e) for e in ids1.ravel())
    keep = []
    arrs = {}
    for which in ("gate", "up", "down"):
        ptrs = (ctypes.c_void_p * E)()
        for e in sorted(need):
            m = np.ascontiguousarray(expert(which, e), dtype=np.uint8)
            keep.append(m)
            ptrs[e] = m.ctypes.data
        arrs[which] = ptrs
    sh = [None if a is None else np.ascontiguousarray(a, dtype=np.uint16) for a in shared]
    g = np.ascontiguousarray(grid, dtype=np.uint8)
    wr = np.ascontiguousarray(wr, dtype=np.uint16)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    L = _Layer(shape.d, shape.f, E, k, shape.f_shared if sh[0] is not None else 0,
               FMT_CODE[shape.fmt_gate], FMT_CODE[shape.fmt_up], FMT_CODE[shape.fmt_down],
               arrs["gate"], arrs["up"], arrs["down"], _ptr(g), _ptr(sh[0]), _ptr(sh[1]), _ptr(sh[2]),
               _ptr(wr), _ptr(b))
    out = np.empty((T, shape.d), np.float64)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    gap = np.empty(T, np.float64)
    nt = nthreads or os.cpu_count() or 1
    rc = lib().orc_layer_forward(ctypes.byref(L), _ptr(x), T, int(alt), nt, _ptr(ids), _ptr(w), _ptr(gap),
                                 _ptr(out))
    if rc != 0:
        raise ValueError("oracle layer failed with status %d" % rc)
    return out, ids, w, gap
