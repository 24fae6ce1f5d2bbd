"""ctypes binding of libds4moe.so (include/ds4moe.h), argument marshalling only.

Tensors are torch CUDA tensors; every call runs on the current torch stream.
Nothing here computes any part of the layer: each step runs in the library's
kernels, and a missing library raises instead of falling back.  Each tensor
argument is checked before the call (on the current CUDA device, contiguous,
the element size and shape or size the call reads or writes), since the
library itself sees only plain pointers.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

from . import synth

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libds4moe.so")

FMT = {"iq2x": 0, "q2k": 1, "q4k": 2, "bf16": 3}
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "CUDA error", 4: "workspace too small",
          5: "device wait timed out", 6: "device-side data error"}

EXPORTS = ["ds4moe_status_string", "ds4moe_prepared_bytes", "ds4moe_prepare", "ds4moe_dequant",
           "ds4moe_route_workspace_size", "ds4moe_route", "ds4moe_workspace_size", "ds4moe_expert_ffn_decode",
           "ds4moe_expert_ffn_grouped", "ds4moe_combine", "ds4moe_last_device_error", "ds4moe_decode_gateup",
           "ds4moe_decode_down", "ds4moe_expert_ffn_decode_noalloc", "ds4moe_selftest_wait_timeout",
           "ds4moe_expert_ffn_grouped_fused"]


class Ds4moeError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("%s failed: %s (%d)" % (what, STATUS.get(code, "?"), code))
        self.code = code


class Experts(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("f", ctypes.c_int32), ("E", ctypes.c_int32), ("f_shared", ctypes.c_int32),
                ("fmt_gate", ctypes.c_int32), ("fmt_up", ctypes.c_int32), ("fmt_down", ctypes.c_int32),
                ("gate", ctypes.c_void_p), ("up", ctypes.c_void_p), ("down", ctypes.c_void_p),
                ("gate_stride", ctypes.c_uint64), ("up_stride", ctypes.c_uint64), ("down_stride", ctypes.c_uint64),
                ("codebook", ctypes.c_void_p),
                ("sh_gate", ctypes.c_void_p), ("sh_up", ctypes.c_void_p), ("sh_down", ctypes.c_void_p)]


_lib = None


def lib():
    """Load the library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libds4moe.so is missing: run `python -m bit_quantized_moe_02_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        vp, i32, u64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_size_t
        l.ds4moe_status_string.restype = ctypes.c_char_p
        l.ds4moe_status_string.argtypes = [i32]
        l.ds4moe_prepared_bytes.restype = sz
        l.ds4moe_prepared_bytes.argtypes = [i32, i32, i32]
        l.ds4moe_prepare.argtypes = [i32, vp, vp, i32, i32, i32, u64, vp]
        l.ds4moe_dequant.argtypes = [i32, vp, vp, i32, i32, vp, vp]
        l.ds4moe_route_workspace_size.restype = sz
        l.ds4moe_route_workspace_size.argtypes = [i32, i32, i32]
        l.ds4moe_route.argtypes = [vp, i32, i32, vp, vp, i32, i32, vp, vp, vp, sz, vp]
        l.ds4moe_workspace_size.restype = sz
        l.ds4moe_workspace_size.argtypes = [ctypes.POINTER(Experts), i32, i32]
        l.ds4moe_expert_ffn_decode.argtypes = [ctypes.POINTER(Experts), vp, i32, vp, vp, i32, vp, vp, sz, vp]
        l.ds4moe_expert_ffn_grouped.argtypes = [ctypes.POINTER(Experts), vp, i32, vp, vp, i32, vp, vp, vp, vp, sz,
                                                vp]
        l.ds4moe_expert_ffn_grouped_fused.argtypes = [ctypes.POINTER(Experts), vp, i32, vp, vp, i32, vp, vp, sz, vp]
        l.ds4moe_combine.argtypes = [vp, vp, vp, i32, i32, i32, vp, vp]
        l.ds4moe_last_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
        l.ds4moe_decode_gateup.argtypes = [ctypes.POINTER(Experts), vp, vp, i32, vp, sz, vp]
        l.ds4moe_decode_down.argtypes = [ctypes.POINTER(Experts), vp, vp, i32, vp, vp, sz, vp]
        l.ds4moe_expert_ffn_decode_noalloc.argtypes = [ctypes.POINTER(Experts), vp, vp, vp, i32, vp, vp]
        l.ds4moe_selftest_wait_timeout.argtypes = [vp]
        _lib = l
    return _lib


def _check(code: int, what: str) -> None:
    if code != 0:
        raise Ds4moeError(code, what)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _arg(t: Optional[torch.Tensor], what: str, dev: int, esize: int, shape=None, numel: Optional[int] = None,
         optional: bool = False):
    """Pointer of a tensor argument after the checks the library cannot make on a plain pointer: a contiguous
    tensor on the current CUDA device, of the element size and shape (or at least the element count) the call
    reads or writes.  A host tensor or a short buffer raises here instead of reaching the kernels."""
    if t is None:
        if optional:
            return None
        raise ValueError("%s: a tensor is required" % what)
    if not t.is_cuda or t.device.index != dev:
        raise ValueError("%s: expected a tensor on the current CUDA device (cuda:%d), got %s" % (what, dev, t.device))
    if not t.is_contiguous():
        raise ValueError("%s: expected a contiguous tensor" % what)
    if t.element_size() != esize:
        raise ValueError("%s: expected %d-byte elements, got %s" % (what, esize, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s: expected shape %s, got %s" % (what, tuple(shape), tuple(t.shape)))
    if numel is not None and t.numel() < numel:
        raise ValueError("%s: expected at least %d elements, got %d" % (what, numel, t.numel()))
    return ctypes.c_void_p(t.data_ptr())


def _bytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


def _cur() -> int:
    return torch.cuda.current_device()


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


# ---- thin wrappers, one per C entry point ----------------------------------------------------------------

def prepared_bytes(fmt: str, rows: int, cols: int) -> int:
    return int(lib().ds4moe_prepared_bytes(FMT[fmt], rows, cols))


def prepare(fmt: str, canonical: torch.Tensor, rows: int, cols: int, n_mats: int,
            out: Optional[torch.Tensor] = None) -> torch.Tensor:
    stride = (prepared_bytes(fmt, rows, cols) + 255) // 256 * 256
    if out is None:
        out = torch.empty(stride * max(n_mats, 1), dtype=torch.uint8, device=canonical.device)
    dev = _cur()
    nbytes = n_mats * rows * (cols // 256) * synth.BLOCK_BYTES.get(fmt, 0)
    pc = _arg(canonical, "prepare: canonical", dev, 1, numel=nbytes)
    po = _arg(out, "prepare: out", dev, 1, numel=stride * n_mats)
    _check(lib().ds4moe_prepare(FMT[fmt], pc, po, rows, cols, n_mats, stride, _stream()), "prepare")
    return out


def dequant(fmt: str, prepared: torch.Tensor, codebook: Optional[torch.Tensor], rows: int, cols: int) -> torch.Tensor:
    out = torch.empty((rows, cols), dtype=torch.float32, device=prepared.device)
    dev = _cur()
    pp = _arg(prepared, "dequant: prepared", dev, 1, numel=prepared_bytes(fmt, rows, cols))
    pg = _arg(codebook, "dequant: codebook", dev, 1, numel=256 * 8, optional=fmt != "iq2x")
    _check(lib().ds4moe_dequant(FMT[fmt], pp, pg, rows, cols, _p(out), _stream()), "dequant")
    return out


def route(x: torch.Tensor, wr: torch.Tensor, bias: Optional[torch.Tensor], k: int, ws: Optional[torch.Tensor] = None,
          ids: Optional[torch.Tensor] = None, weights: Optional[torch.Tensor] = None):
    T, d = x.shape
    E = wr.shape[0]
    if ws is None:  # a caller-provided workspace is checked against the required size by the library
        ws = torch.empty(max(int(lib().ds4moe_route_workspace_size(T, d, E)), 1), dtype=torch.uint8, device=x.device)
    ids = torch.empty((T, k), dtype=torch.int32, device=x.device) if ids is None else ids
    weights = torch.empty((T, k), dtype=torch.float32, device=x.device) if weights is None else weights
    dev = _cur()
    px = _arg(x, "route: x", dev, 2)
    pw = _arg(wr, "route: w_router", dev, 2, shape=(E, d))
    pb = _arg(bias, "route: bias", dev, 4, shape=(E,), optional=True)
    pi = _arg(ids, "route: ids", dev, 4, shape=(T, k))
    pr = _arg(weights, "route: weights", dev, 4, shape=(T, k))
    ps = _arg(ws, "route: workspace", dev, ws.element_size())
    _check(lib().ds4moe_route(px, T, d, pw, pb, E, k, pi, pr, ps, _bytes(ws), _stream()), "route")
    return ids, weights


def workspace_size(ex: Experts, T: int, k: int) -> int:
    return int(lib().ds4moe_workspace_size(ctypes.byref(ex), T, k))


def expert_ffn_decode(ex: Experts, x: torch.Tensor, ids: torch.Tensor, weights: torch.Tensor, ws: torch.Tensor,
                      out: Optional[torch.Tensor] = None) -> torch.Tensor:
    B, k = ids.shape
    out = torch.empty((B, ex.d), dtype=torch.float32, device=x.device) if out is None else out
    dev = _cur()
    px = _arg(x, "expert_ffn_decode: x", dev, 2, shape=(B, ex.d))
    pi = _arg(ids, "expert_ffn_decode: ids", dev, 4)
    pr = _arg(weights, "expert_ffn_decode: weights", dev, 4, shape=(B, k))
    po = _arg(out, "expert_ffn_decode: out", dev, 4, shape=(B, ex.d))
    ps = _arg(ws, "expert_ffn_decode: workspace", dev, ws.element_size())
    _check(lib().ds4moe_expert_ffn_decode(ctypes.byref(ex), px, B, pi, pr, k, po, ps, _bytes(ws), _stream()),
           "expert_ffn_decode")
    return out


def decode_gateup(ex: Experts, x: torch.Tensor, ids: torch.Tensor, ws: torch.Tensor) -> None:
    k = ids.shape[-1]
    dev = _cur()
    px = _arg(x, "decode_gateup: x", dev, 2, numel=ex.d)
    pi = _arg(ids, "decode_gateup: ids", dev, 4, numel=k)
    ps = _arg(ws, "decode_gateup: workspace", dev, ws.element_size())
    _check(lib().ds4moe_decode_gateup(ctypes.byref(ex), px, pi, k, ps, _bytes(ws), _stream()), "decode_gateup")


def decode_down(ex: Experts, ids: torch.Tensor, weights: torch.Tensor, ws: torch.Tensor, out: torch.Tensor) -> None:
    k = ids.shape[-1]
    dev = _cur()
    pi = _arg(ids, "decode_down: ids", dev, 4, numel=k)
    pr = _arg(weights, "decode_down: weights", dev, 4, numel=k)
    po = _arg(out, "decode_down: out", dev, 4, numel=ex.d)
    ps = _arg(ws, "decode_down: workspace", dev, ws.element_size())
    _check(lib().ds4moe_decode_down(ctypes.byref(ex), pi, pr, k, po, ps, _bytes(ws), _stream()), "decode_down")


def expert_ffn_decode_noalloc(ex: Experts, x: torch.Tensor, ids: torch.Tensor, weights: torch.Tensor,
                              out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """B = 1 decode served from the library's fixed scratch array (no workspace argument)."""
    out = torch.empty((1, ex.d), dtype=torch.float32, device=x.device) if out is None else out
    k = ids.shape[-1]
    dev = _cur()
    px = _arg(x, "expert_ffn_decode_noalloc: x", dev, 2, numel=ex.d)
    pi = _arg(ids, "expert_ffn_decode_noalloc: ids", dev, 4, numel=k)
    pr = _arg(weights, "expert_ffn_decode_noalloc: weights", dev, 4, numel=k)
    po = _arg(out, "expert_ffn_decode_noalloc: out", dev, 4, numel=ex.d)
    _check(lib().ds4moe_expert_ffn_decode_noalloc(ctypes.byref(ex), px, pi, pr, k, po, _stream()),
           "expert_ffn_decode_noalloc")
    return out


def expert_ffn_grouped(ex: Experts, x: torch.Tensor, ids: torch.Tensor, weights: torch.Tensor, ws: torch.Tensor,
                       y_perm: torch.Tensor, inv_perm: torch.Tensor, y_shared: Optional[torch.Tensor]) -> None:
    T, k = ids.shape
    dev = _cur()
    px = _arg(x, "expert_ffn_grouped: x", dev, 2, shape=(T, ex.d))
    pi = _arg(ids, "expert_ffn_grouped: ids", dev, 4)
    pr = _arg(weights, "expert_ffn_grouped: weights", dev, 4, shape=(T, k))
    py = _arg(y_perm, "expert_ffn_grouped: y_perm", dev, 4, numel=T * k * ex.d)
    pv = _arg(inv_perm, "expert_ffn_grouped: inv_perm", dev, 4, numel=T * k)
    pz = _arg(y_shared, "expert_ffn_grouped: y_shared", dev, 4, numel=T * ex.d, optional=True)
    ps = _arg(ws, "expert_ffn_grouped: workspace", dev, ws.element_size())
    _check(lib().ds4moe_expert_ffn_grouped(ctypes.byref(ex), px, T, pi, pr, k, py, pv, pz, ps, _bytes(ws),
                                           _stream()), "expert_ffn_grouped")


def expert_ffn_grouped_fused(ex: Experts, x: torch.Tensor, ids: torch.Tensor, weights: torch.Tensor,
                             ws: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Prefill with the combine fused into the down GEMM: returns the layer output [T, d] (fp32)."""
    T, k = ids.shape
    out = torch.empty((T, ex.d), dtype=torch.float32, device=x.device) if out is None else out
    dev = _cur()
    px = _arg(x, "expert_ffn_grouped_fused: x", dev, 2, shape=(T, ex.d))
    pi = _arg(ids, "expert_ffn_grouped_fused: ids", dev, 4)
    pr = _arg(weights, "expert_ffn_grouped_fused: weights", dev, 4, shape=(T, k))
    po = _arg(out, "expert_ffn_grouped_fused: out", dev, 4, numel=T * ex.d)
    ps = _arg(ws, "expert_ffn_grouped_fused: workspace", dev, ws.element_size())
    _check(lib().ds4moe_expert_ffn_grouped_fused(ctypes.byref(ex), px, T, pi, pr, k, po, ps, _bytes(ws),
                                                 _stream()), "expert_ffn_grouped_fused")
    return out


def combine(y_perm: torch.Tensor, inv_perm: torch.Tensor, y_shared: Optional[torch.Tensor], T: int, d: int, k: int,
            out: Optional[torch.Tensor] = None) -> torch.Tensor:
    out = torch.empty((T, d), dtype=torch.float32, device=y_perm.device) if out is None else out
    dev = _cur()
    py = _arg(y_perm, "combine: y_perm", dev, 4, numel=T * k * d)
    pv = _arg(inv_perm, "combine: inv_perm", dev, 4, numel=T * k)
    pz = _arg(y_shared, "combine: y_shared", dev, 4, numel=T * d, optional=True)
    po = _arg(out, "combine: out", dev, 4, numel=T * d)
    _check(lib().ds4moe_combine(py, pv, pz, T, d, k, po, _stream()), "combine")
    return out


def last_device_error() -> int:
    code = ctypes.c_int32(0)
    _check(lib().ds4moe_last_device_error(_stream(), ctypes.byref(code)), "last_device_error")
    return int(code.value)


# ---- a layer held on the device ------------------------------------------------------------------------------

class DeviceLayer:
    """One MoE FFN layer resident in HBM: prepared expert planes, codebook, router, shared expert.

    ``forward(x)`` runs route -> experts -> combine for any number of tokens: T = 1 takes the decode GEMV path,
    larger T the permuted grouped path.  All buffers, including the workspace, are allocated here once.
    """

    def __init__(self, host: "synth.Layer", device="cuda", max_tokens: int = 1):
        s = host.shape
        self.shape = s
        self.device = torch.device(device)
        dev = self.device

        def up(a):
            return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

        self.wr = up(host.wr).view(torch.float16)
        self.bias = up(host.bias) if np.any(host.bias != 0) else None
        self.codebook = up(host.grid.reshape(-1))
        self.planes = {}
        strides = {}
        for which, fmt, rows, cols in (("gate", s.fmt_gate, s.f, s.d), ("up", s.fmt_up, s.f, s.d),
                                       ("down", s.fmt_down, s.d, s.f)):
            stride = (prepared_bytes(fmt, rows, cols) + 255) // 256 * 256
            buf = torch.empty(stride * s.E, dtype=torch.uint8, device=dev)
            chunk = 16  # experts uploaded per canonical staging copy
            for e0 in range(0, s.E, chunk):
                e1 = min(s.E, e0 + chunk)
                canon = up(np.stack([host.expert(which, e) for e in range(e0, e1)]))
                prepare(fmt, canon, rows, cols, e1 - e0, out=buf[e0 * stride:])
                del canon
            self.planes[which] = buf
            strides[which] = stride
        host.drop_cache()
        self.sh = [None if a is None else up(a).view(torch.bfloat16) for a in (host.sh_gate, host.sh_up,
                                                                                host.sh_down)]
        fs = s.f_shared if self.sh[0] is not None else 0
        self.ex = Experts(s.d, s.f, s.E, fs, FMT[s.fmt_gate], FMT[s.fmt_up], FMT[s.fmt_down],
                          self.planes["gate"].data_ptr(), self.planes["up"].data_ptr(),
                          self.planes["down"].data_ptr(), strides["gate"], strides["up"], strides["down"],
                          self.codebook.data_ptr(),
                          self.sh[0].data_ptr() if fs else None, self.sh[1].data_ptr() if fs else None,
                          self.sh[2].data_ptr() if fs else None)
        self.max_tokens = 0
        self.reserve(max_tokens)

    def reserve(self, T: int) -> None:
        if T <= self.max_tokens:
            return
        s = self.shape
        need = max(workspace_size(self.ex, T, s.k), 1)
        self.ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        self.route_ws = torch.empty(max(int(lib().ds4moe_route_workspace_size(T, s.d, s.E)), 1), dtype=torch.uint8,
                                    device=self.device)
        self.ids_buf = torch.empty((T, s.k), dtype=torch.int32, device=self.device)
        self.w_buf = torch.empty((T, s.k), dtype=torch.float32, device=self.device)
        self.max_tokens = T

    def route(self, x: torch.Tensor, ids: Optional[torch.Tensor] = None, weights: Optional[torch.Tensor] = None):
        return route(x, self.wr, self.bias, self.shape.k, ws=self.route_ws, ids=ids, weights=weights)

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, return_routing: bool = False):
        """Layer output for x [T, d] (bf16): route, experts, combine.  Without return_routing the routing goes
        to buffers owned by the layer (reused by the next call on the same stream order)."""
        T = x.shape[0]
        self.reserve(T)
        if return_routing:
            ids, w = self.route(x)
        else:
            ids, w = self.route(x, ids=self.ids_buf[:T], weights=self.w_buf[:T])
        out = expert_ffn_decode(self.ex, x, ids, w, self.ws, out=out)
        return (out, ids, w) if return_routing else out

    def decode_graph(self, host_io: bool = False) -> "DecodeGraph":
        """A CUDA-graph replay of this layer's single-token decode (route + experts); see DecodeGraph."""
        return DecodeGraph(self, host_io=host_io)

    def forward_grouped(self, x: torch.Tensor):
        """Prefill entry: grouped experts then combine (returns out, ids, weights, y_perm, inv_perm)."""
        s = self.shape
        T = x.shape[0]
        self.reserve(T)
        ids, w = self.route(x)
        y_perm = torch.empty((T * s.k, s.d), dtype=torch.float32, device=x.device)
        inv = torch.empty(T * s.k, dtype=torch.int32, device=x.device)
        ys = torch.empty((T, s.d), dtype=torch.float32, device=x.device) if self.ex.f_shared else None
        expert_ffn_grouped(self.ex, x, ids, w, self.ws, y_perm, inv, ys)
        out = combine(y_perm, inv, ys, T, s.d, s.k)
        return out, ids, w, y_perm, inv

    def forward_fused(self, x: torch.Tensor, out: Optional[torch.Tensor] = None):
        """Prefill entry with the combine fused into the down GEMM (returns out, ids, weights).  The k routed
        rows of a token are summed by atomic adds, in no fixed order."""
        T = x.shape[0]
        self.reserve(T)
        ids, w = self.route(x, ids=self.ids_buf[:T], weights=self.w_buf[:T])
        out = expert_ffn_grouped_fused(self.ex, x, ids, w, self.ws, out=out)
        return out, ids, w


class DecodeGraph:
    """Single-token decode of one layer replayed from a CUDA graph: the router, top-k, gate/up and down launches
    of ``DeviceLayer.forward`` for one token, captured once, so a decode step costs one graph launch on the host.

    ``x`` (bf16 [1, d]) and ``out`` (fp32 [1, d]) are buffers owned by this object: write the token into ``x``
    (or pass it to ``__call__``), replay, read ``out``.  Replays run on the current stream; consecutive replays
    reuse the same buffers, so read ``out`` before the next one.

    With ``host_io=True`` the graph also holds the two copies: it starts with a copy of the pinned host buffer
    ``x_host`` (int16 bits of the bf16 token) to the device and ends with a copy of the output to the pinned host
    buffer ``out_host``, so a decode step from host memory to host memory is one graph launch.  ``__call__``
    then writes its argument into ``x_host`` (a host copy) and returns ``out_host``, which holds the result once
    the stream has been synchronized; write the next token only after that synchronization.
    """

    def __init__(self, layer: DeviceLayer, host_io: bool = False):
        s = layer.shape
        dev = layer.device
        self.layer = layer
        self.x = torch.zeros((1, s.d), dtype=torch.bfloat16, device=dev)
        self.out = torch.empty((1, s.d), dtype=torch.float32, device=dev)
        self.ids = torch.empty((1, s.k), dtype=torch.int32, device=dev)
        self.weights = torch.empty((1, s.k), dtype=torch.float32, device=dev)
        # workspaces of its own: the graph keeps their addresses, which a later layer.reserve() must not free
        self.ws = torch.empty(max(workspace_size(layer.ex, 1, s.k), 1), dtype=torch.uint8, device=dev)
        self.route_ws = torch.empty(max(int(lib().ds4moe_route_workspace_size(1, s.d, s.E)), 1), dtype=torch.uint8,
                                    device=dev)
        self.host_io = host_io
        if host_io:
            self.x_host = torch.zeros((1, s.d), dtype=torch.int16).pin_memory()
            self.out_host = torch.zeros((1, s.d), dtype=torch.float32).pin_memory()
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            self._record()  # eager run first: the library configures its kernels outside the capture
            side.synchronize()
            self.graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.graph, stream=side):
                self._record()
        torch.cuda.current_stream(dev).wait_stream(side)

    def _record(self):
        L = self.layer
        if self.host_io:
            self.x.view(torch.int16).copy_(self.x_host, non_blocking=True)
        route(self.x, L.wr, L.bias, L.shape.k, ws=self.route_ws, ids=self.ids, weights=self.weights)
        expert_ffn_decode(L.ex, self.x, self.ids, self.weights, self.ws, out=self.out)
        if self.host_io:
            self.out_host.copy_(self.out, non_blocking=True)

    def __call__(self, x: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Copy x (bf16 or int16 bits, [1, d], device or pinned host) into the input buffer if given, replay,
        and return the output buffer."""
        if self.host_io:
            if x is not None:
                self.x_host.copy_(x.view(torch.int16))
            self.graph.replay()
            return self.out_host
        if x is not None:
            self.x.view(torch.int16).copy_(x.view(torch.int16), non_blocking=True)
        self.graph.replay()
        return self.out
