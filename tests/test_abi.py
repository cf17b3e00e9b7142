"""The C-ABI library without a GPU: it loads, exports every symbol the headers
declare, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

import precision_quantization_row_b200 as nv
from precision_quantization_row_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return nv.lib()


def _declared(paths):
    names = []
    for path in paths:
        with open(path) as f:
            names += re.findall(r"NVFP4PT_API\s+[\w\s\*]+?\b(nvfp4pt_\w+)\s*\(", f.read())
    return names


def _exported(lib_path):
    """Names of the dynamic symbols a shared library defines (nm -D --defined-only)."""
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], check=True, capture_output=True, text=True).stdout
    return {line.split()[-1] for line in out.splitlines() if line.strip()}


def test_every_declared_symbol_is_exported(L):
    names = _declared([os.path.join(ROOT, "include", h) for h in ("nvfp4pt.h", "nvfp4pt_timing.h")])
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(nv.EXPORTS)
    # the product library exports the C ABI of the headers and nothing else of ours
    ours = {s for s in _exported(nv.LIB_PATH) if s.startswith("nvfp4pt")}
    assert ours == set(names)


def test_probe_library_exports_apart():
    """The diagnostic probes live in their own test-only library."""
    import probe
    lib_path = probe.build()
    names = _declared([os.path.join(ROOT, "tests", "probe", "nvfp4pt_probe.h")])
    assert set(names) == set(probe.EXPORTS)
    ours = {s for s in _exported(lib_path) if s.startswith("nvfp4pt")}
    assert ours == set(names)
    assert not any(n.startswith("nvfp4pt_probe") for n in _exported(nv.LIB_PATH))


def test_status_strings(L):
    for code in range(9):
        assert L.nvfp4pt_status_string(code)
    assert L.nvfp4pt_status_string(99) == b"unknown status"


def test_workspace_bytes(L):
    # error word + observed maxima + bf16 column maxima [groups, cols]
    assert nv.workspace_bytes(16, 16, 1) >= 20 + 2 * 16
    assert nv.workspace_bytes(65536, 7168, 64) >= 16 + 4 * 64 + 2 * 64 * 7168
    assert nv.workspace_bytes(16, 16, 1024) >= 16 + 4 * 1024 + 2 * 1024 * 16
    assert nv.workspace_bytes(16384, 8192, 1) >= 16 + 4 + 2 * 8192
    assert nv.workspace_bytes(16, 16, 7) % 256 == 0


class _Host:
    """A 16-byte aligned host scratch area standing in for pointers (never dereferenced:
    every call below fails validation before any device access)."""

    def __init__(self):
        self.buf = ctypes.create_string_buffer(1 << 12)
        self.a = (ctypes.addressof(self.buf) + 15) // 16 * 16

    def p(self, off=0):
        return ctypes.c_void_p(self.a + off)


F0 = ctypes.c_float(0.0)


def test_quantize_rejections(L):
    h = _Host()
    P = h.p
    q = lambda x, r, c, fl, *o: L.nvfp4pt_quantize(x, r, c, fl, *o, None, F0, P(), None)
    ok7 = [P()] * 6
    assert q(None, 16, 16, 3, *ok7) == 1
    assert q(P(), 16, 16, 1, None, P(), P(), None, None, None) == 1            # rowwise output missing
    assert q(P(), 16, 16, 2, P(), P(), P(), P(), None, P()) == 1                # colwise output missing
    assert L.nvfp4pt_quantize(P(), 16, 16, 3, *ok7, None, F0, None, None) == 1  # workspace
    for r, c in [(15, 16), (16, 8), (0, 16), (16, -16), (1 << 31, 16), (96, 70), (70, 96)]:
        assert q(P(), r, c, 3, *ok7) == 2, (r, c)
    for fl in (0, 4, 7):
        assert q(P(), 16, 16, fl, *ok7) == 7, fl
    assert q(P(8), 16, 16, 3, *ok7) == 3
    assert q(P(), 16, 16, 3, P(4), P(), P(), P(), P(), P()) == 3
    assert q(P(), 16, 16, 3, P(), P(), P(), P(), P(), P(2)) == 3
    assert L.nvfp4pt_quantize(P(), 16, 16, 3, *ok7, P(4), F0, P(), None) == 3  # absmax buffer alignment
    # rowwise only: columnwise pointers are ignored, even if misaligned
    assert q(P(), 16, 16, 1, P(), P(), P(), P(3), None, None) not in (1, 3)


def test_grouped_rejections(L):
    h = _Host()
    P = h.p

    def g(offs, G=None, rows=64):
        arr = (ctypes.c_int64 * len(offs))(*offs)
        G = len(offs) - 1 if G is None else G
        return L.nvfp4pt_quantize_grouped(P(), rows, 32, arr, G, 3, *[P()] * 6, None, F0, P(), None)

    assert L.nvfp4pt_quantize_grouped(P(), 64, 32, None, 1, 3, *[P()] * 6, None, F0, P(), None) == 1
    assert g([0, 64], G=0) == 4
    assert g([0, 64], G=1025) == 4
    assert g([16, 64]) == 4          # does not start at 0
    assert g([0, 48]) == 4           # does not end at rows
    assert g([0, 32, 16, 64]) == 4   # decreasing
    assert g([0, 8, 64]) == 4        # not a multiple of 16
    # valid offsets (including empty groups) pass validation and fail only at the CUDA step here
    assert g([0, 0, 32, 32, 64]) in (5, 6)


def test_weight_and_absmax_rejections(L):
    h = _Host()
    P = h.p
    assert L.nvfp4pt_quantize_weight_2d(None, 16, 16, P(), P(), P(), P(), None) == 1
    assert L.nvfp4pt_quantize_weight_2d(P(), 16, 17, P(), P(), P(), P(), None) == 2
    assert L.nvfp4pt_quantize_weight_2d(P(), 16, 16, P(1), P(), P(), P(), None) == 3
    assert L.nvfp4pt_update_absmax(None, P(), 4, F0, None) == 1
    assert L.nvfp4pt_update_absmax(P(), None, 4, F0, None) == 1
    assert L.nvfp4pt_update_absmax(P(), P(), -1, F0, None) == 2
    assert L.nvfp4pt_update_absmax(P(2), P(), 4, F0, None) == 3
    assert L.nvfp4pt_workspace_error(None, None, None) == 1


def test_dequant_and_requant_rejections(L):
    h = _Host()
    P = h.p
    d = L.nvfp4pt_dequantize
    assert d(None, P(), P(), 16, 16, P(), None) == 1
    assert d(P(), P(), P(), 16, 16, None, None) == 1
    assert d(P(), P(), P(), 16, 24, P(), None) == 2
    assert d(P(), P(8), P(), 16, 16, P(), None) == 3
    assert d(P(), P(), P(), 16, 16, P(4), None) == 3
    # the rows' decode scales, then a cast workspace, at any width
    for cols in (16, 16400):
        assert (L.nvfp4pt_requantize_workspace_bytes(16, cols, 1) ==
                256 + L.nvfp4pt_workspace_bytes(16, cols, 1))
    assert L.nvfp4pt_requantize_workspace_bytes(1024, 64, 3) == 4096 + L.nvfp4pt_workspace_bytes(1024, 64, 3)

    def r(*args, offs=None, G=1, rows=64, ws=None):
        arr = None if offs is None else (ctypes.c_int64 * len(offs))(*offs)
        a = list(args) if args else [P()] * 3
        return L.nvfp4pt_requantize_colwise(*a, rows, 32, arr, G, P(), P(), P(), None, F0,
                                            P() if ws is None else ws, None)

    assert r(None, P(), P()) == 1
    assert L.nvfp4pt_requantize_colwise(P(), P(), P(), 64, 32, None, 1, P(), P(), P(), None, F0, None, None) == 1
    assert L.nvfp4pt_requantize_colwise(P(), P(), P(), 64, 20, None, 1, P(), P(), P(), None, F0, P(), None) == 2
    assert r(P(), P(), P(2)) == 3
    assert r(offs=[0, 8, 64], G=2) == 4
    assert r(offs=[0, 64], G=0) == 4
    # valid (ungrouped and grouped) pass validation and fail only at the device step here
    assert r() in (5, 6)
    assert r(offs=[0, 0, 32, 64], G=3) in (5, 6)


def test_gemm_rejections(L):
    h = _Host()
    P = h.p
    g = lambda qa=None, m=128, n=256, k=512, d=None, ws=None, sfb=None: L.nvfp4pt_gemm_per_token(
        P() if qa is None else qa, P(), P(), m, P(), P() if sfb is None else sfb, P(), n, k,
        P() if d is None else d, P() if ws is None else ws, None)
    # the error word, then both operands' block scales (rows padded to 128 for A, 256 for B)
    assert L.nvfp4pt_gemm_workspace_bytes(16, 16, 256) == 256 + 128 * 16 + 256 * 16
    assert L.nvfp4pt_gemm_workspace_bytes(16384, 8192, 8192) == 256 + (16384 + 8192) * 512
    assert L.nvfp4pt_gemm_workspace_bytes(-1, 16, 256) == 256
    assert L.nvfp4pt_gemm_per_token(None, P(), P(), 16, P(), P(), P(), 16, 256, P(), P(), None) == 1
    assert L.nvfp4pt_gemm_per_token(P(), P(), P(), 16, P(), P(), P(), 16, 256, None, P(), None) == 1
    assert L.nvfp4pt_gemm_per_token(P(), P(), P(), 16, P(), P(), P(), 16, 256, P(), None, None) == 1
    for m, n, k in [(0, 16, 256), (16, 8, 256), (20, 16, 256), (16, 16, 128), (16, 16, 300), (16, 16, 0),
                    (1 << 31, 16, 256)]:
        assert g(m=m, n=n, k=k) == 2, (m, n, k)
    assert g(qa=P(8)) == 3
    assert g(sfb=P(4)) == 3
    assert g(d=P(4)) == 3
    # valid arguments pass validation and fail only at the device step here
    assert g() in (5, 6)


def test_options_rejections(L):
    import precision_quantization_row_b200 as nvp
    h = _Host()
    P = h.p

    def o(flags=0, cols=32, rows=64, opt_flags=nvp.COL_RHT):
        arr = (ctypes.c_int64 * 2)(0, rows)
        opts = nvp.ColwiseOptions(opt_flags, 0xBEEF, 1, 2)
        return L.nvfp4pt_quantize_grouped_opts(P(), rows, cols, arr, 1, flags or 3, *[P()] * 6, None, F0,
                                               ctypes.byref(opts), P(), None)

    assert o(opt_flags=4) == 7
    assert o(opt_flags=8) == 7
    assert o(cols=16400) == 2                       # options need rows of at most 16384 elements
    assert o(cols=16400, flags=1) in (5, 6)         # ... only for the columnwise direction
    assert o(cols=20) == 2
    assert o() in (5, 6)
    assert o(opt_flags=3) in (5, 6)
    assert L.nvfp4pt_quantize_grouped_opts(P(), 64, 32, (ctypes.c_int64 * 2)(0, 64), 1, 3, *[P()] * 6, None, F0,
                                           None, P(), None) in (5, 6)   # NULL options: the plain cast


def test_probe_rejections():
    import probe
    PL = probe.lib()
    h = _Host()
    P = h.p
    assert PL.nvfp4pt_probe_transitions(0, None, 8, P(), None) == 1
    assert PL.nvfp4pt_probe_transitions(2, P(), 8, P(), None) == 7
    assert PL.nvfp4pt_probe_pairs(P(), 0, P(), None) == 2


def test_noalloc_rejections(L):
    """The entry without allocation reports argument errors as the grouped cast does,
    before any CUDA call (here, on a machine without a GPU, nothing else can run)."""
    h = _Host()
    P = h.p

    def n(offs=(0, 64), G=None, rows=64, cols=32, flags=3, outs=None, x=None, bufs=None):
        arr = None if offs is None else (ctypes.c_int64 * len(offs))(*offs)
        G = len(offs) - 1 if G is None else G
        o = [P()] * 6 if outs is None else outs
        return L.nvfp4pt_quantize_grouped_noalloc(P() if x is None else x, rows, cols, arr, G, flags, *o, bufs, F0,
                                                  None)

    assert L.nvfp4pt_quantize_grouped_noalloc(None, 64, 32, (ctypes.c_int64 * 2)(0, 64), 1, 3, *[P()] * 6, None,
                                              F0, None) == 1
    assert n(offs=None, G=1) == 1
    assert n(flags=1, outs=[None, P(), P(), None, None, None]) == 1      # rowwise output missing
    assert n(flags=2, outs=[None, None, None, P(), P(), None]) == 1      # colwise output missing
    for r, c in [(15, 16), (16, 8), (0, 16), (1 << 31, 16), (96, 70)]:
        assert n(offs=(0, max(r, 0)), rows=r, cols=c) == 2, (r, c)
    for fl in (0, 4, 7):
        assert n(flags=fl) == 7, fl
    assert n(x=P(8)) == 3
    assert n(outs=[P(4), P(), P(), P(), P(), P()]) == 3
    assert n(bufs=P(4)) == 3
    assert n(offs=(0, 64), G=0) == 4
    assert n(offs=(16, 64)) == 4
    assert n(offs=(0, 32, 16, 64)) == 4
    assert n(offs=(0, 8, 64)) == 4
    # more groups than the static array holds (NVFP4PT_NOALLOC_MAX_GROUPS = 252)
    offs = tuple(range(0, 16 * 253 + 1, 16))
    assert n(offs=offs, rows=16 * 253) == 4
    # valid arguments pass validation and fail only at the device step here
    assert n(offs=(0, 0, 32, 64)) in (5, 6)


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros((16, 16), dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        nv.quantize(x)
    with pytest.raises(TypeError):
        nv.quantize_weight_2d(x)
