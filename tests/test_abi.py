"""The C-ABI library loads without a GPU, exports every symbol the header declares, and its host-side checks
reject bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

from bit_quantized_moe_02_b200 import ds4moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    src = open(os.path.join(ROOT, "include", "ds4moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ds4moe_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_header_symbol():
    lib = ds4moe.lib()
    syms = header_symbols()
    assert len(syms) >= 13
    for s in syms:
        assert hasattr(lib, s), s
    assert sorted(ds4moe.EXPORTS) == [s for s in syms if s in ds4moe.EXPORTS]


def test_status_strings():
    lib = ds4moe.lib()
    for code in range(7):
        assert lib.ds4moe_status_string(code)
    assert lib.ds4moe_status_string(99) == b"unknown status"


def test_prepared_bytes_layout():
    # planes rounded to 256 B: IQ2X 32+32+4+2 B per block, Q2K 64+16+4, Q4K 128+12+4
    def r(x):
        return (x + 255) // 256 * 256
    for rows, cols in ((1, 256), (512, 256), (2048, 4096), (4096, 2048), (3, 768)):
        n = rows * cols // 256
        assert ds4moe.prepared_bytes("iq2x", rows, cols) == r(32 * n) * 2 + r(4 * n) + r(2 * n)
        assert ds4moe.prepared_bytes("q2k", rows, cols) == r(64 * n) + r(16 * n) + r(4 * n)
        assert ds4moe.prepared_bytes("q4k", rows, cols) == r(128 * n) + r(12 * n) + r(4 * n)
    assert ds4moe.prepared_bytes("iq2x", 4, 100) == 0
    assert ds4moe.prepared_bytes("bf16", 4, 256) == 0


def test_host_side_argument_checks():
    lib = ds4moe.lib()
    vp = ctypes.c_void_p
    fake = vp(1 << 20)  # never dereferenced: every call below fails its host checks first
    assert lib.ds4moe_prepare(0, None, fake, 4, 256, 1, 4096, None) == 1
    assert lib.ds4moe_prepare(0, fake, fake, 4, 100, 1, 4096, None) == 1
    assert lib.ds4moe_prepare(3, fake, fake, 4, 256, 1, 4096, None) == 2
    assert lib.ds4moe_prepare(0, fake, vp((1 << 20) + 16), 4, 256, 1, 4096, None) == 1  # unaligned planes
    assert lib.ds4moe_prepare(0, fake, fake, 4, 256, 1, 256, None) == 1  # stride below prepared size
    assert lib.ds4moe_route(fake, 1, 256, fake, None, 8, 9, fake, fake, fake, 1 << 20, None) == 1  # k > E
    assert lib.ds4moe_route(fake, 1, 256, fake, None, 2048, 2, fake, fake, fake, 1 << 20, None) == 1  # E > 1024
    assert lib.ds4moe_route(fake, 1, 256, fake, None, 8, 2, fake, fake, fake, 4, None) == 4  # workspace
    assert lib.ds4moe_route(None, 0, 256, None, None, 8, 2, None, None, None, 0, None) == 0  # T = 0: no-op
    assert lib.ds4moe_combine(fake, fake, None, 1, 10, 2, fake, None) == 1  # d % 4
    ex = ds4moe.Experts(256, 512, 8, 0, 0, 0, 1, 1 << 20, 1 << 21, 1 << 22, 1 << 16, 1 << 16, 1 << 16, 1 << 23,
                        None, None, None)
    assert lib.ds4moe_workspace_size(ctypes.byref(ex), 1, 2) > 0
    bad = ds4moe.Experts(*[getattr(ex, f) for f, _ in ds4moe.Experts._fields_])
    bad.fmt_up = 2
    assert lib.ds4moe_workspace_size(ctypes.byref(bad), 1, 2) == 0
    assert lib.ds4moe_expert_ffn_decode(ctypes.byref(bad), fake, 1, fake, fake, 2, fake, fake, 1 << 30, None) == 2
    assert lib.ds4moe_expert_ffn_decode(ctypes.byref(ex), fake, 1, fake, fake, 2, fake, fake, 16, None) == 4
    bad.fmt_up = 0
    bad.gate_stride = 1000
    assert lib.ds4moe_expert_ffn_grouped(ctypes.byref(bad), fake, 4, fake, fake, 2, fake, fake, None, fake, 1 << 30,
                                         None) == 1
    bad.gate_stride = 1 << 16
    bad.f_shared = 256  # shared expert without weights
    assert lib.ds4moe_expert_ffn_grouped(ctypes.byref(bad), fake, 4, fake, fake, 2, fake, fake, None, fake, 1 << 30,
                                         None) == 1
    # fused-combine prefill: missing output, misaligned output, short workspace
    assert lib.ds4moe_expert_ffn_grouped_fused(ctypes.byref(ex), fake, 4, fake, fake, 2, None, fake, 1 << 30,
                                               None) == 1
    assert lib.ds4moe_expert_ffn_grouped_fused(ctypes.byref(ex), fake, 4, fake, fake, 2, ctypes.c_void_p((1 << 20) + 4),
                                               fake, 1 << 30, None) == 1
    assert lib.ds4moe_expert_ffn_grouped_fused(ctypes.byref(ex), fake, 4, fake, fake, 2, fake, fake, 16, None) == 4
    assert lib.ds4moe_last_device_error(None, None) == 1


def test_decode_gemv_limits_checked_on_host():
    """The single-token GEMV halves refuse layers outside their limits before any launch: d and f 256 times a power
    of two up to 8192, IQ2X gate/up with Q2K down or Q4K throughout, k <= 32; the combined decode call then runs
    the grouped path instead (its own checks)."""
    lib = ds4moe.lib()
    fake = ctypes.c_void_p(1 << 20)

    def experts(d, f, fmt_gate=0, fmt_down=1, fs=0):
        return ds4moe.Experts(d, f, 8, fs, fmt_gate, fmt_gate, fmt_down, 1 << 20, 1 << 22, 1 << 24, 1 << 26,
                              1 << 26, 1 << 26, 1 << 23, None, None, None)

    for d, f in ((768, 512), (256, 768), (16384, 512)):  # not 256 * 2^i, or d beyond 8192
        ex = experts(d, f)
        assert lib.ds4moe_decode_gateup(ctypes.byref(ex), fake, fake, 2, fake, 1 << 30, None) == 2, (d, f)
        assert lib.ds4moe_decode_down(ctypes.byref(ex), fake, fake, 2, fake, fake, 1 << 30, None) == 2, (d, f)
    mixed = experts(512, 512, fmt_gate=2, fmt_down=1)  # Q4K gate/up with Q2K down: no GEMV kernel pair
    assert lib.ds4moe_decode_gateup(ctypes.byref(mixed), fake, fake, 2, fake, 1 << 30, None) == 2
    mixed = experts(512, 512, fmt_gate=0, fmt_down=2)  # IQ2X gate/up with Q4K down
    assert lib.ds4moe_decode_down(ctypes.byref(mixed), fake, fake, 2, fake, fake, 1 << 30, None) == 2
    ex = experts(512, 512)
    assert lib.ds4moe_decode_gateup(ctypes.byref(ex), fake, fake, 40, fake, 1 << 30, None) == 1  # k > E
    # workspace: h (k*f floats) and the shared expert's h, each rounded to 256 bytes
    need = (2 * 512 * 4 + 255) // 256 * 256 + 256
    assert lib.ds4moe_decode_gateup(ctypes.byref(ex), fake, fake, 2, fake, need - 1, None) == 4
    assert lib.ds4moe_expert_ffn_decode_noalloc(ctypes.byref(experts(768, 512)), fake, fake, fake, 2, fake,
                                                None) == 2


def test_grouped_path_expert_limit():
    """The grouped path's offset scan is one CTA of 1024 threads: more than 1024 experts are refused before any
    launch (and the workspace query returns 0) for the batches that need that path, while the GEMV path (batches
    of up to 16 tokens), which has no such scan, still takes such a layer."""
    lib = ds4moe.lib()
    fake = ctypes.c_void_p(1 << 20)
    big = ds4moe.Experts(256, 512, 2048, 0, 0, 0, 1, 1 << 20, 1 << 21, 1 << 22, 1 << 16, 1 << 16, 1 << 16, 1 << 23,
                         None, None, None)
    assert lib.ds4moe_workspace_size(ctypes.byref(big), 17, 2) == 0  # B > 16: grouped path only
    assert lib.ds4moe_workspace_size(ctypes.byref(big), 1, 2) > 0  # B <= 16: GEMV path
    assert lib.ds4moe_workspace_size(ctypes.byref(big), 16, 2) > 0
    assert lib.ds4moe_expert_ffn_grouped(ctypes.byref(big), fake, 4, fake, fake, 2, fake, fake, None, fake,
                                         1 << 30, None) == 1
    assert lib.ds4moe_expert_ffn_grouped_fused(ctypes.byref(big), fake, 4, fake, fake, 2, fake, fake, 1 << 30,
                                               None) == 1
    assert lib.ds4moe_expert_ffn_decode(ctypes.byref(big), fake, 17, fake, fake, 2, fake, fake, 1 << 30, None) == 1
    mixed = ds4moe.Experts(256, 512, 2048, 0, 2, 2, 1, 1 << 20, 1 << 21, 1 << 22, 1 << 17, 1 << 17, 1 << 17, None,
                           None, None, None)  # Q4K gate/up with Q2K down: even B = 1 needs the grouped path
    assert lib.ds4moe_workspace_size(ctypes.byref(mixed), 1, 2) == 0
    assert lib.ds4moe_expert_ffn_decode(ctypes.byref(mixed), fake, 1, fake, fake, 2, fake, fake, 1 << 30,
                                        None) == 1


def test_empty_inputs_are_no_ops():
    """Zero tokens: every many-token entry point returns OK without touching its (absent) buffers."""
    lib = ds4moe.lib()
    ex = ds4moe.Experts(256, 512, 8, 0, 0, 0, 1, 1 << 20, 1 << 21, 1 << 22, 1 << 16, 1 << 16, 1 << 16, 1 << 23,
                        None, None, None)
    assert lib.ds4moe_route(None, 0, 256, None, None, 8, 2, None, None, None, 0, None) == 0
    assert lib.ds4moe_expert_ffn_decode(ctypes.byref(ex), None, 0, None, None, 2, None, None, 0, None) == 0
    assert lib.ds4moe_expert_ffn_grouped(ctypes.byref(ex), None, 0, None, None, 2, None, None, None, None, 0,
                                         None) == 0
    assert lib.ds4moe_expert_ffn_grouped_fused(ctypes.byref(ex), None, 0, None, None, 2, None, None, 0, None) == 0
    assert lib.ds4moe_combine(None, None, None, 0, 256, 2, None, None) == 0
    # negative counts are errors, not no-ops
    assert lib.ds4moe_expert_ffn_decode(ctypes.byref(ex), None, -1, None, None, 2, None, None, 0, None) == 1
    assert lib.ds4moe_expert_ffn_grouped(ctypes.byref(ex), None, -1, None, None, 2, None, None, None, None, 0,
                                         None) == 1
    assert lib.ds4moe_expert_ffn_grouped_fused(ctypes.byref(ex), None, -1, None, None, 2, None, None, 0,
                                               None) == 1
    assert lib.ds4moe_combine(None, None, None, -1, 256, 2, None, None) == 1
