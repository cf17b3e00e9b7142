"""B200 (sm_100a) NVFP4 per-token quantization cast: Python binding of libnvfp4pt.

Thin ctypes marshalling over the C ABI in include/nvfp4pt.h. Every step of the cast
runs in the library's CUDA kernels; PyTorch only provides device memory and the
current stream. There is no CPU fallback: a missing library or a non-CUDA tensor
raises.

    out = quantize(x)                       # x: bf16 CUDA [rows, cols]
    out["q_row"], out["sf_row"], out["amax_row"], out["q_col"], ...

Names follow the C entry points (nvfp4pt_quantize -> quantize, ...).
"""
from __future__ import annotations

import ctypes
import functools
import os

import torch

ROWWISE = 1
COLWISE = 2
MAX_GROUPS = 1024
NOALLOC_MAX_GROUPS = 252   # NVFP4PT_NOALLOC_MAX_GROUPS

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4pt.so")

STATUS = {
    0: "NVFP4PT_OK", 1: "NVFP4PT_ERR_NULL", 2: "NVFP4PT_ERR_SHAPE", 3: "NVFP4PT_ERR_ALIGN",
    4: "NVFP4PT_ERR_GROUPS", 5: "NVFP4PT_ERR_ARCH", 6: "NVFP4PT_ERR_CUDA", 7: "NVFP4PT_ERR_FLAGS",
    8: "NVFP4PT_ERR_DEVICE",
}

EXPORTS = (
    "nvfp4pt_status_string", "nvfp4pt_workspace_bytes", "nvfp4pt_quantize", "nvfp4pt_quantize_grouped",
    "nvfp4pt_quantize_weight_2d", "nvfp4pt_update_absmax", "nvfp4pt_workspace_error",
    "nvfp4pt_quantize_grouped_noalloc", "nvfp4pt_quantize_timed", "nvfp4pt_dequantize", "nvfp4pt_requantize_workspace_bytes",
    "nvfp4pt_requantize_colwise", "nvfp4pt_gemm_workspace_bytes", "nvfp4pt_gemm_per_token",
    "nvfp4pt_quantize_grouped_opts",
)

COL_RHT = 1   # NVFP4PT_COL_RHT
COL_SR = 2    # NVFP4PT_COL_SR


class ColwiseOptions(ctypes.Structure):
    """nvfp4pt_colwise_options."""
    _fields_ = [("flags", ctypes.c_int), ("rht_signs", ctypes.c_uint32), ("sr_seed", ctypes.c_uint64),
                ("sr_offset", ctypes.c_uint64)]


class Nvfp4ptError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn}: {STATUS.get(status, status)} ({text})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libnvfp4pt.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m precision_quantization_row_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        L.nvfp4pt_status_string.argtypes, L.nvfp4pt_status_string.restype = [I], ctypes.c_char_p
        L.nvfp4pt_workspace_bytes.argtypes, L.nvfp4pt_workspace_bytes.restype = [I64, I64, I], ctypes.c_size_t
        L.nvfp4pt_quantize.argtypes = [P, I64, I64, I, P, P, P, P, P, P, P, F, P, P]
        L.nvfp4pt_quantize_grouped.argtypes = [P, I64, I64, P, I, I, P, P, P, P, P, P, P, F, P, P]
        L.nvfp4pt_quantize_weight_2d.argtypes = [P, I64, I64, P, P, P, P, P]
        L.nvfp4pt_update_absmax.argtypes = [P, P, I64, F, P]
        L.nvfp4pt_workspace_error.argtypes = [P, P, P]
        L.nvfp4pt_quantize_grouped_noalloc.argtypes = [P, I64, I64, P, I, I, P, P, P, P, P, P, P, F, P]
        L.nvfp4pt_quantize_timed.argtypes = [P, I64, I64, I, P, P, P, P, P, P, P, F, P, P, P]
        L.nvfp4pt_dequantize.argtypes = [P, P, P, I64, I64, P, P]
        L.nvfp4pt_requantize_workspace_bytes.argtypes = [I64, I64, I]
        L.nvfp4pt_requantize_colwise.argtypes = [P, P, P, I64, I64, P, I, P, P, P, P, F, P, P]
        L.nvfp4pt_quantize_grouped_opts.argtypes = [P, I64, I64, P, I, I, P, P, P, P, P, P, P, F, P, P, P]
        L.nvfp4pt_gemm_workspace_bytes.argtypes = [I64, I64, I64]
        L.nvfp4pt_gemm_per_token.argtypes = [P, P, P, I64, P, P, P, I64, I64, P, P, P]
        for name in EXPORTS[2:]:
            getattr(L, name).restype = I
        L.nvfp4pt_requantize_workspace_bytes.restype = ctypes.c_size_t
        L.nvfp4pt_gemm_workspace_bytes.restype = ctypes.c_size_t
        _lib = L
    return _lib


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise Nvfp4ptError(fn, status, lib().nvfp4pt_status_string(status).decode())


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream, device):
    s = torch.cuda.current_stream(device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _require_2d(x, name: str, dtype) -> None:
    if not isinstance(x, torch.Tensor) or x.dtype != dtype or x.dim() != 2 or not x.is_contiguous():
        raise TypeError(f"{name} must be a contiguous 2D {dtype} tensor")


def _require_cuda(x: torch.Tensor, name: str) -> None:
    if not x.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (there is no CPU path)")


# The C ABI takes raw pointers and cannot see buffer sizes, so the binding checks what
# the kernels rely on before any call: each buffer's dtype, contiguity, element count
# and device (that of the call's main input; CPU tensors meet the same checks, and the
# main input's "must be CUDA" check comes last).
def _buf(t, name: str, dtype, n: int, dev: int) -> int:
    try:
        if t.dtype is dtype and t.numel() >= n and t.is_contiguous() and t.get_device() == dev:
            return t.data_ptr()
    except AttributeError:   # not a tensor
        pass
    raise _bad_buf(t, name, dtype, n, dev)


def _bad_buf(t, name: str, dtype, n: int, dev: int) -> Exception:
    if not isinstance(t, torch.Tensor):
        return TypeError(f"{name} must be a torch.Tensor")
    if t.dtype is not dtype:
        return TypeError(f"{name} must be {dtype}, not {t.dtype}")
    if not t.is_contiguous():
        return ValueError(f"{name} must be contiguous")
    if t.numel() < n:
        return ValueError(f"{name} holds {t.numel()} elements, the call needs {n}")
    return TypeError(f"{name} is on device {t.get_device()}, the call's input on {dev}")


def _out_ptrs(out: dict, flags: int, rows: int, cols: int, groups: int, dev: int) -> list:
    """Pointers of the cast's outputs for `flags` (None for the direction not asked for)."""
    p = [None] * 6
    if flags & ROWWISE:
        p[0] = _buf(out.get("q_row"), "q_row", torch.uint8, rows * cols // 2, dev)
        p[1] = _buf(out.get("sf_row"), "sf_row", torch.uint8, rows * cols // 16, dev)
        p[2] = _buf(out.get("amax_row"), "amax_row", torch.float32, rows, dev)
    if flags & COLWISE:
        p[3] = _buf(out.get("q_col"), "q_col", torch.uint8, cols * rows // 2, dev)
        p[4] = _buf(out.get("sf_col"), "sf_col", torch.uint8, cols * rows // 16, dev)
        p[5] = _buf(out.get("amax_col"), "amax_col", torch.float32, groups * cols, dev)
    return p


def _opt_buf(t, name: str, dtype, n: int, dev: int):
    return None if t is None else _buf(t, name, dtype, n, dev)


@functools.lru_cache(maxsize=256)
def workspace_bytes(rows: int, cols: int, num_groups: int = 1) -> int:
    return int(lib().nvfp4pt_workspace_bytes(rows, cols, num_groups))


def new_workspace(rows: int, cols: int, num_groups: int = 1, device=None) -> torch.Tensor:
    return torch.empty(workspace_bytes(rows, cols, num_groups), dtype=torch.uint8, device=device)


def _outputs(rows, cols, flags, device, col_rows=None, groups=1):
    out = {}
    if flags & ROWWISE:
        out["q_row"] = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
        out["sf_row"] = torch.empty((rows, cols // 16), dtype=torch.uint8, device=device)
        out["amax_row"] = torch.empty(rows, dtype=torch.float32, device=device)
    if flags & COLWISE:
        if groups == 1 and col_rows is None:
            out["q_col"] = torch.empty((cols, rows // 2), dtype=torch.uint8, device=device)
            out["sf_col"] = torch.empty((cols, rows // 16), dtype=torch.uint8, device=device)
            out["amax_col"] = torch.empty(cols, dtype=torch.float32, device=device)
        else:  # grouped: flat per-group column blocks
            out["q_col"] = torch.empty(cols * rows // 2, dtype=torch.uint8, device=device)
            out["sf_col"] = torch.empty(cols * rows // 16, dtype=torch.uint8, device=device)
            out["amax_col"] = torch.empty((groups, cols), dtype=torch.float32, device=device)
    return out


def quantize(x: torch.Tensor, flags: int = ROWWISE | COLWISE, absmax: torch.Tensor | None = None,
             decay: float = 0.0, out: dict | None = None, workspace: torch.Tensor | None = None,
             stream: torch.cuda.Stream | None = None) -> dict:
    """nvfp4pt_quantize. absmax: optional fp32 CUDA tensor of one element, updated in place."""
    _require_2d(x, "x", torch.bfloat16)
    rows, cols = x.shape
    dev = x.get_device()
    out = _outputs(rows, cols, flags, x.device) if out is None else out
    ws = new_workspace(rows, cols, 1, x.device) if workspace is None else workspace
    p = _out_ptrs(out, flags, rows, cols, 1, dev)
    pa = _opt_buf(absmax, "absmax", torch.float32, 1, dev)
    pw = _buf(ws, "workspace", torch.uint8, workspace_bytes(rows, cols, 1), dev)
    _require_cuda(x, "x")
    st = lib().nvfp4pt_quantize(_ptr(x), rows, cols, flags, *p, pa, ctypes.c_float(decay), pw,
                                _stream(stream, x.device))
    _check("nvfp4pt_quantize", st)
    return out


CAST_LAUNCHES = 3   # kernel launches of one quantize call (nvfp4pt_timing.h)


def quantize_timed(x: torch.Tensor, events, flags: int = ROWWISE | COLWISE, absmax: torch.Tensor | None = None,
                   decay: float = 0.0, out: dict | None = None, workspace: torch.Tensor | None = None,
                   stream: torch.cuda.Stream | None = None) -> dict:
    """nvfp4pt_quantize_timed: quantize with events[0] recorded before the first kernel
    launch and events[i] after the i-th (CAST_LAUNCHES + 1 torch.cuda.Event objects,
    created with enable_timing=True and already recorded once, so that they exist)."""
    _require_2d(x, "x", torch.bfloat16)
    if len(events) != CAST_LAUNCHES + 1:
        raise ValueError(f"need {CAST_LAUNCHES + 1} events")
    rows, cols = x.shape
    dev = x.get_device()
    out = _outputs(rows, cols, flags, x.device) if out is None else out
    ws = new_workspace(rows, cols, 1, x.device) if workspace is None else workspace
    p = _out_ptrs(out, flags, rows, cols, 1, dev)
    pa = _opt_buf(absmax, "absmax", torch.float32, 1, dev)
    pw = _buf(ws, "workspace", torch.uint8, workspace_bytes(rows, cols, 1), dev)
    _require_cuda(x, "x")
    if any(e.cuda_event == 0 for e in events):
        raise ValueError("every event must have been recorded once (torch creates it lazily)")
    evs = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    st = lib().nvfp4pt_quantize_timed(_ptr(x), rows, cols, flags, *p, pa, ctypes.c_float(decay), pw,
                                      _stream(stream, x.device), evs)
    _check("nvfp4pt_quantize_timed", st)
    return out


def dequantize(q: torch.Tensor, sf: torch.Tensor, amax: torch.Tensor, out: torch.Tensor | None = None,
               stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """nvfp4pt_dequantize: rowwise-layout NVFP4 data (q uint8 [rows, cols/2], sf uint8
    [rows, cols/16], amax fp32 [rows]) back to bf16 [rows, cols]."""
    _require_2d(q, "q", torch.uint8)
    rows, half = q.shape
    cols = 2 * half
    dev = q.get_device()
    ps = _buf(sf, "sf", torch.uint8, rows * cols // 16, dev)
    pa = _buf(amax, "amax", torch.float32, rows, dev)
    out = torch.empty((rows, cols), dtype=torch.bfloat16, device=q.device) if out is None else out
    po = _buf(out, "out", torch.bfloat16, rows * cols, dev)
    _require_cuda(q, "q")
    st = lib().nvfp4pt_dequantize(_ptr(q), ps, pa, rows, cols, po, _stream(stream, q.device))
    _check("nvfp4pt_dequantize", st)
    return out


def gemm_per_token(qa: torch.Tensor, sfa: torch.Tensor, amax_a: torch.Tensor, qb: torch.Tensor,
                   sfb: torch.Tensor, amax_b: torch.Tensor, out: torch.Tensor | None = None,
                   workspace: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """nvfp4pt_gemm_per_token: D [m, n] fp32 of two K-major rowwise NVFP4 operands (A: q
    uint8 [m, k/2], sf uint8 [m, k/16], amax fp32 [m]; B likewise with n rows), rescaled by
    S_dec(amax_a[m]) * S_dec(amax_b[n]) in the epilogue."""
    _require_2d(qa, "qa", torch.uint8)
    _require_2d(qb, "qb", torch.uint8)
    m, half = qa.shape
    n = qb.shape[0]
    k = 2 * half
    if qb.shape[1] != half:
        raise ValueError(f"qa and qb differ in K: {qa.shape} vs {qb.shape}")
    dev = qa.get_device()
    psa = _buf(sfa, "sfa", torch.uint8, m * k // 16, dev)
    paa = _buf(amax_a, "amax_a", torch.float32, m, dev)
    pqb = _buf(qb, "qb", torch.uint8, n * k // 2, dev)
    psb = _buf(sfb, "sfb", torch.uint8, n * k // 16, dev)
    pab = _buf(amax_b, "amax_b", torch.float32, n, dev)
    out = torch.empty((m, n), dtype=torch.float32, device=qa.device) if out is None else out
    po = _buf(out, "out", torch.float32, m * n, dev)
    ws = new_gemm_workspace(m, n, k, qa.device) if workspace is None else workspace
    pw = _buf(ws, "workspace", torch.uint8, gemm_workspace_bytes(m, n, k), dev)
    _require_cuda(qa, "qa")
    st = lib().nvfp4pt_gemm_per_token(_ptr(qa), psa, paa, m, pqb, psb, pab, n, k, po, pw,
                                      _stream(stream, qa.device))
    _check("nvfp4pt_gemm_per_token", st)
    return out


@functools.lru_cache(maxsize=256)
def gemm_workspace_bytes(m: int, n: int, k: int) -> int:
    return int(lib().nvfp4pt_gemm_workspace_bytes(m, n, k))


def new_gemm_workspace(m: int, n: int, k: int, device=None) -> torch.Tensor:
    return torch.empty(gemm_workspace_bytes(m, n, k), dtype=torch.uint8, device=device)


@functools.lru_cache(maxsize=256)
def requantize_workspace_bytes(rows: int, cols: int, groups: int = 1) -> int:
    return int(lib().nvfp4pt_requantize_workspace_bytes(rows, cols, groups))


def requantize_colwise(q_row: torch.Tensor, sf_row: torch.Tensor, amax_row: torch.Tensor, offsets=None,
                       absmax: torch.Tensor | None = None, decay: float = 0.0, out: dict | None = None,
                       workspace: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None) -> dict:
    """nvfp4pt_requantize_colwise: the columnwise outputs (q_col, sf_col, amax_col) of the
    cast of the dequantized rowwise data; offsets: None or the host row offsets of the
    token groups."""
    _require_2d(q_row, "q_row", torch.uint8)
    rows, half = q_row.shape
    cols = 2 * half
    dev = q_row.get_device()
    ps = _buf(sf_row, "sf_row", torch.uint8, rows * cols // 16, dev)
    pa = _buf(amax_row, "amax_row", torch.float32, rows, dev)
    G = 1 if offsets is None else len(offsets) - 1
    if out is None:
        d = q_row.device
        if offsets is None:
            out = {"q_col": torch.empty((cols, rows // 2), dtype=torch.uint8, device=d),
                   "sf_col": torch.empty((cols, rows // 16), dtype=torch.uint8, device=d),
                   "amax_col": torch.empty(cols, dtype=torch.float32, device=d)}
        else:
            out = {"q_col": torch.empty(cols * rows // 2, dtype=torch.uint8, device=d),
                   "sf_col": torch.empty(cols * rows // 16, dtype=torch.uint8, device=d),
                   "amax_col": torch.empty((G, cols), dtype=torch.float32, device=d)}
    if workspace is None:
        workspace = torch.empty(requantize_workspace_bytes(rows, cols, G), dtype=torch.uint8, device=q_row.device)
    p = _out_ptrs(out, COLWISE, rows, cols, max(G, 1), dev)
    pb = _opt_buf(absmax, "absmax", torch.float32, max(G, 1), dev)
    pw = _buf(workspace, "workspace", torch.uint8, requantize_workspace_bytes(rows, cols, max(G, 1)), dev)
    _require_cuda(q_row, "q_row")
    off = None if offsets is None else (ctypes.c_int64 * len(offsets))(*[int(o) for o in offsets])
    st = lib().nvfp4pt_requantize_colwise(_ptr(q_row), ps, pa, rows, cols, off, G, p[3], p[4], p[5], pb,
                                          ctypes.c_float(decay), pw, _stream(stream, q_row.device))
    _check("nvfp4pt_requantize_colwise", st)
    return out


def quantize_grouped(x: torch.Tensor, offsets, flags: int = ROWWISE | COLWISE, absmax: torch.Tensor | None = None,
                     decay: float = 0.0, out: dict | None = None, workspace: torch.Tensor | None = None,
                     stream: torch.cuda.Stream | None = None) -> dict:
    """nvfp4pt_quantize_grouped. offsets: host sequence of num_groups+1 row offsets."""
    _require_2d(x, "x", torch.bfloat16)
    rows, cols = x.shape
    dev = x.get_device()
    off = (ctypes.c_int64 * len(offsets))(*[int(o) for o in offsets])
    G = len(offsets) - 1
    out = _outputs(rows, cols, flags, x.device, col_rows=rows, groups=G) if out is None else out
    ws = new_workspace(rows, cols, max(G, 1), x.device) if workspace is None else workspace
    p = _out_ptrs(out, flags, rows, cols, max(G, 1), dev)
    pa = _opt_buf(absmax, "absmax", torch.float32, max(G, 1), dev)
    pw = _buf(ws, "workspace", torch.uint8, workspace_bytes(rows, cols, max(G, 1)), dev)
    _require_cuda(x, "x")
    st = lib().nvfp4pt_quantize_grouped(_ptr(x), rows, cols, off, G, flags, *p, pa, ctypes.c_float(decay), pw,
                                        _stream(stream, x.device))
    _check("nvfp4pt_quantize_grouped", st)
    return out


def quantize_grouped_opts(x: torch.Tensor, offsets=None, flags: int = ROWWISE | COLWISE,
                          absmax: torch.Tensor | None = None, decay: float = 0.0, rht: bool = False,
                          rht_signs: int = 0, sr: bool = False, seed: int = 0, offset: int = 0,
                          out: dict | None = None, workspace: torch.Tensor | None = None,
                          stream: torch.cuda.Stream | None = None) -> dict:
    """nvfp4pt_quantize_grouped_opts: the cast with the columnwise options (the Hadamard
    transform of each columnwise 16-row block with the sign mask rht_signs; stochastic
    rounding with the Philox seed and offset). offsets None: one group, and the outputs
    are shaped as quantize's."""
    _require_2d(x, "x", torch.bfloat16)
    rows, cols = x.shape
    dev = x.get_device()
    offs = [0, rows] if offsets is None else list(offsets)
    off = (ctypes.c_int64 * len(offs))(*[int(o) for o in offs])
    G = len(offs) - 1
    if out is None:
        out = _outputs(rows, cols, flags, x.device) if offsets is None else \
            _outputs(rows, cols, flags, x.device, col_rows=rows, groups=G)
    ws = new_workspace(rows, cols, max(G, 1), x.device) if workspace is None else workspace
    p = _out_ptrs(out, flags, rows, cols, max(G, 1), dev)
    pa = _opt_buf(absmax, "absmax", torch.float32, max(G, 1), dev)
    pw = _buf(ws, "workspace", torch.uint8, workspace_bytes(rows, cols, max(G, 1)), dev)
    _require_cuda(x, "x")
    opts = ColwiseOptions((COL_RHT if rht else 0) | (COL_SR if sr else 0), rht_signs & 0xFFFF,
                          seed & (2**64 - 1), offset & (2**64 - 1))
    st = lib().nvfp4pt_quantize_grouped_opts(_ptr(x), rows, cols, off, G, flags, *p, pa, ctypes.c_float(decay),
                                             ctypes.byref(opts), pw, _stream(stream, x.device))
    _check("nvfp4pt_quantize_grouped_opts", st)
    return out


def quantize_grouped_noalloc(x: torch.Tensor, offsets, flags: int = ROWWISE | COLWISE,
                             absmax: torch.Tensor | None = None, decay: float = 0.0, out: dict | None = None,
                             stream: torch.cuda.Stream | None = None) -> dict:
    """nvfp4pt_quantize_grouped_noalloc: the grouped cast without a workspace (its scratch
    is a static array in the library; at most NOALLOC_MAX_GROUPS token groups). The
    outputs are allocated here when `out` is None; pass `out` to allocate nothing."""
    _require_2d(x, "x", torch.bfloat16)
    rows, cols = x.shape
    dev = x.get_device()
    off = (ctypes.c_int64 * len(offsets))(*[int(o) for o in offsets])
    G = len(offsets) - 1
    out = _outputs(rows, cols, flags, x.device, col_rows=rows, groups=G) if out is None else out
    p = _out_ptrs(out, flags, rows, cols, max(G, 1), dev)
    pa = _opt_buf(absmax, "absmax", torch.float32, max(G, 1), dev)
    _require_cuda(x, "x")
    st = lib().nvfp4pt_quantize_grouped_noalloc(_ptr(x), rows, cols, off, G, flags, *p, pa, ctypes.c_float(decay),
                                                _stream(stream, x.device))
    _check("nvfp4pt_quantize_grouped_noalloc", st)
    return out


def quantize_weight_2d(w: torch.Tensor, out: dict | None = None, workspace: torch.Tensor | None = None,
                       stream: torch.cuda.Stream | None = None) -> dict:
    """nvfp4pt_quantize_weight_2d (rowwise outputs with 16x16-block scales)."""
    _require_2d(w, "w", torch.bfloat16)
    rows, cols = w.shape
    dev = w.get_device()
    out = _outputs(rows, cols, ROWWISE, w.device) if out is None else out
    ws = new_workspace(rows, cols, 1, w.device) if workspace is None else workspace
    p = _out_ptrs(out, ROWWISE, rows, cols, 1, dev)
    pw = _buf(ws, "workspace", torch.uint8, workspace_bytes(rows, cols, 1), dev)
    _require_cuda(w, "w")
    st = lib().nvfp4pt_quantize_weight_2d(_ptr(w), rows, cols, p[0], p[1], p[2], pw, _stream(stream, w.device))
    _check("nvfp4pt_quantize_weight_2d", st)
    return out


def update_absmax(absmax: torch.Tensor, amax_vec: torch.Tensor, decay: float,
                  stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """nvfp4pt_update_absmax: absmax[0] = max(absmax[0] * decay, max(amax_vec)), in place."""
    dev = absmax.get_device() if isinstance(absmax, torch.Tensor) else -1
    pb = _buf(absmax, "absmax", torch.float32, 1, dev)
    pv = _buf(amax_vec, "amax_vec", torch.float32, 0, dev)
    _require_cuda(absmax, "absmax")
    st = lib().nvfp4pt_update_absmax(pb, pv, amax_vec.numel(), ctypes.c_float(decay), _stream(stream, absmax.device))
    _check("nvfp4pt_update_absmax", st)
    return absmax


def workspace_error(workspace: torch.Tensor, stream: torch.cuda.Stream | None = None) -> int:
    """The device error word of the last call on this workspace (synchronises the stream)."""
    word = ctypes.c_uint32(0)
    dev = workspace.get_device() if isinstance(workspace, torch.Tensor) else -1
    pw = _buf(workspace, "workspace", torch.uint8, 4, dev)
    _require_cuda(workspace, "workspace")
    st = lib().nvfp4pt_workspace_error(pw, ctypes.byref(word), _stream(stream, workspace.device))
    if st not in (0, 8):
        _check("nvfp4pt_workspace_error", st)
    return int(word.value)
