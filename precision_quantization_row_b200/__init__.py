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
import os

import torch

ROWWISE = 1
COLWISE = 2
MAX_GROUPS = 1024

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
    "nvfp4pt_probe_transitions", "nvfp4pt_probe_pairs", "nvfp4pt_probe_e4m3_decode", "nvfp4pt_probe_div6",
    "nvfp4pt_probe_e4m3_div", "nvfp4pt_quantize_grouped_noalloc", "nvfp4pt_probe_pair_scales",
    "nvfp4pt_quantize_timed", "nvfp4pt_dequantize", "nvfp4pt_requantize_workspace_bytes",
    "nvfp4pt_requantize_colwise",
)


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
        L.nvfp4pt_probe_transitions.argtypes = [I, P, ctypes.c_uint32, P, P]
        L.nvfp4pt_probe_pairs.argtypes = [P, I64, P, P]
        L.nvfp4pt_probe_e4m3_decode.argtypes = [P, P]
        L.nvfp4pt_probe_div6.argtypes = [P, P]
        L.nvfp4pt_probe_e4m3_div.argtypes = [I, I, P, P]
        L.nvfp4pt_quantize_grouped_noalloc.argtypes = [P, I64, I64, P, I, I, P, P, P, P, P, P, P, F, P]
        L.nvfp4pt_probe_pair_scales.argtypes = [I, I, ctypes.c_uint32, P, P]
        L.nvfp4pt_quantize_timed.argtypes = [P, I64, I64, I, P, P, P, P, P, P, P, F, P, P, P]
        L.nvfp4pt_dequantize.argtypes = [P, P, P, I64, I64, P, P]
        L.nvfp4pt_requantize_workspace_bytes.argtypes = [I64, I64, I]
        L.nvfp4pt_requantize_colwise.argtypes = [P, P, P, I64, I64, P, I, P, P, P, P, F, P, P]
        for name in EXPORTS[2:]:
            getattr(L, name).restype = I
        L.nvfp4pt_requantize_workspace_bytes.restype = ctypes.c_size_t
        _lib = L
    return _lib


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise Nvfp4ptError(fn, status, lib().nvfp4pt_status_string(status).decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    s = torch.cuda.current_stream(device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _require_cuda_bf16(x: torch.Tensor, name: str):
    if not isinstance(x, torch.Tensor) or not x.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_contiguous():
        raise TypeError(f"{name} must be a contiguous 2D bfloat16 tensor")


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
    _require_cuda_bf16(x, "x")
    rows, cols = x.shape
    out = _outputs(rows, cols, flags, x.device) if out is None else out
    ws = new_workspace(rows, cols, 1, x.device) if workspace is None else workspace
    st = lib().nvfp4pt_quantize(
        _ptr(x), rows, cols, flags, _ptr(out.get("q_row")), _ptr(out.get("sf_row")), _ptr(out.get("amax_row")),
        _ptr(out.get("q_col")), _ptr(out.get("sf_col")), _ptr(out.get("amax_col")), _ptr(absmax),
        ctypes.c_float(decay), _ptr(ws), _stream(stream, x.device))
    _check("nvfp4pt_quantize", st)
    return out


CAST_LAUNCHES = 3   # kernel launches of one quantize call (nvfp4pt_timing.h)


def quantize_timed(x: torch.Tensor, events, flags: int = ROWWISE | COLWISE, absmax: torch.Tensor | None = None,
                   decay: float = 0.0, out: dict | None = None, workspace: torch.Tensor | None = None,
                   stream: torch.cuda.Stream | None = None) -> dict:
    """nvfp4pt_quantize_timed: quantize with events[0] recorded before the first kernel
    launch and events[i] after the i-th (CAST_LAUNCHES + 1 torch.cuda.Event objects,
    created with enable_timing=True and already recorded once, so that they exist)."""
    _require_cuda_bf16(x, "x")
    if len(events) != CAST_LAUNCHES + 1:
        raise ValueError(f"need {CAST_LAUNCHES + 1} events")
    rows, cols = x.shape
    out = _outputs(rows, cols, flags, x.device) if out is None else out
    ws = new_workspace(rows, cols, 1, x.device) if workspace is None else workspace
    evs = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    st = lib().nvfp4pt_quantize_timed(
        _ptr(x), rows, cols, flags, _ptr(out.get("q_row")), _ptr(out.get("sf_row")), _ptr(out.get("amax_row")),
        _ptr(out.get("q_col")), _ptr(out.get("sf_col")), _ptr(out.get("amax_col")), _ptr(absmax),
        ctypes.c_float(decay), _ptr(ws), _stream(stream, x.device), evs)
    _check("nvfp4pt_quantize_timed", st)
    return out


def dequantize(q: torch.Tensor, sf: torch.Tensor, amax: torch.Tensor, out: torch.Tensor | None = None,
               stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """nvfp4pt_dequantize: rowwise-layout NVFP4 data (q uint8 [rows, cols/2], sf uint8
    [rows, cols/16], amax fp32 [rows]) back to bf16 [rows, cols]."""
    for t, n in ((q, "q"), (sf, "sf"), (amax, "amax")):
        if not t.is_cuda:
            raise ValueError(f"{n} must be a CUDA tensor")
    rows, half = q.shape
    cols = 2 * half
    out = torch.empty((rows, cols), dtype=torch.bfloat16, device=q.device) if out is None else out
    st = lib().nvfp4pt_dequantize(_ptr(q), _ptr(sf), _ptr(amax), rows, cols, _ptr(out), _stream(stream, q.device))
    _check("nvfp4pt_dequantize", st)
    return out


def requantize_workspace_bytes(rows: int, cols: int, groups: int = 1) -> int:
    return int(lib().nvfp4pt_requantize_workspace_bytes(rows, cols, groups))


def requantize_colwise(q_row: torch.Tensor, sf_row: torch.Tensor, amax_row: torch.Tensor, offsets=None,
                       absmax: torch.Tensor | None = None, decay: float = 0.0, out: dict | None = None,
                       workspace: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None) -> dict:
    """nvfp4pt_requantize_colwise: the columnwise outputs (q_col, sf_col, amax_col) of the
    cast of the dequantized rowwise data; offsets: None or the host row offsets of the
    token groups."""
    for t, n in ((q_row, "q_row"), (sf_row, "sf_row"), (amax_row, "amax_row")):
        if not t.is_cuda:
            raise ValueError(f"{n} must be a CUDA tensor")
    rows, half = q_row.shape
    cols = 2 * half
    G = 1 if offsets is None else len(offsets) - 1
    if out is None:
        dev = q_row.device
        if offsets is None:
            out = {"q_col": torch.empty((cols, rows // 2), dtype=torch.uint8, device=dev),
                   "sf_col": torch.empty((cols, rows // 16), dtype=torch.uint8, device=dev),
                   "amax_col": torch.empty(cols, dtype=torch.float32, device=dev)}
        else:
            out = {"q_col": torch.empty(cols * rows // 2, dtype=torch.uint8, device=dev),
                   "sf_col": torch.empty(cols * rows // 16, dtype=torch.uint8, device=dev),
                   "amax_col": torch.empty((G, cols), dtype=torch.float32, device=dev)}
    if workspace is None:
        workspace = torch.empty(requantize_workspace_bytes(rows, cols, G), dtype=torch.uint8, device=q_row.device)
    off = None if offsets is None else (ctypes.c_int64 * len(offsets))(*[int(o) for o in offsets])
    st = lib().nvfp4pt_requantize_colwise(
        _ptr(q_row), _ptr(sf_row), _ptr(amax_row), rows, cols, off, G, _ptr(out["q_col"]), _ptr(out["sf_col"]),
        _ptr(out["amax_col"]), _ptr(absmax), ctypes.c_float(decay), _ptr(workspace), _stream(stream, q_row.device))
    _check("nvfp4pt_requantize_colwise", st)
    return out


def quantize_grouped(x: torch.Tensor, offsets, flags: int = ROWWISE | COLWISE, absmax: torch.Tensor | None = None,
                     decay: float = 0.0, out: dict | None = None, workspace: torch.Tensor | None = None,
                     stream: torch.cuda.Stream | None = None) -> dict:
    """nvfp4pt_quantize_grouped. offsets: host sequence of num_groups+1 row offsets."""
    _require_cuda_bf16(x, "x")
    rows, cols = x.shape
    off = (ctypes.c_int64 * len(offsets))(*[int(o) for o in offsets])
    G = len(offsets) - 1
    out = _outputs(rows, cols, flags, x.device, col_rows=rows, groups=G) if out is None else out
    ws = new_workspace(rows, cols, max(G, 1), x.device) if workspace is None else workspace
    st = lib().nvfp4pt_quantize_grouped(
        _ptr(x), rows, cols, off, G, flags, _ptr(out.get("q_row")), _ptr(out.get("sf_row")),
        _ptr(out.get("amax_row")), _ptr(out.get("q_col")), _ptr(out.get("sf_col")), _ptr(out.get("amax_col")),
        _ptr(absmax), ctypes.c_float(decay), _ptr(ws), _stream(stream, x.device))
    _check("nvfp4pt_quantize_grouped", st)
    return out


def quantize_weight_2d(w: torch.Tensor, out: dict | None = None, workspace: torch.Tensor | None = None,
                       stream: torch.cuda.Stream | None = None) -> dict:
    """nvfp4pt_quantize_weight_2d (rowwise outputs with 16x16-block scales)."""
    _require_cuda_bf16(w, "w")
    rows, cols = w.shape
    out = _outputs(rows, cols, ROWWISE, w.device) if out is None else out
    ws = new_workspace(rows, cols, 1, w.device) if workspace is None else workspace
    st = lib().nvfp4pt_quantize_weight_2d(_ptr(w), rows, cols, _ptr(out["q_row"]), _ptr(out["sf_row"]),
                                          _ptr(out["amax_row"]), _ptr(ws), _stream(stream, w.device))
    _check("nvfp4pt_quantize_weight_2d", st)
    return out


def update_absmax(absmax: torch.Tensor, amax_vec: torch.Tensor, decay: float,
                  stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """nvfp4pt_update_absmax: absmax[0] = max(absmax[0] * decay, max(amax_vec)), in place."""
    if not (absmax.is_cuda and amax_vec.is_cuda) or absmax.dtype != torch.float32 or amax_vec.dtype != torch.float32:
        raise TypeError("absmax and amax_vec must be fp32 CUDA tensors")
    st = lib().nvfp4pt_update_absmax(_ptr(absmax), _ptr(amax_vec), amax_vec.numel(), ctypes.c_float(decay),
                                     _stream(stream, absmax.device))
    _check("nvfp4pt_update_absmax", st)
    return absmax


def workspace_error(workspace: torch.Tensor, stream: torch.cuda.Stream | None = None) -> int:
    """The device error word of the last call on this workspace (synchronises the stream)."""
    word = ctypes.c_uint32(0)
    st = lib().nvfp4pt_workspace_error(_ptr(workspace), ctypes.byref(word), _stream(stream, workspace.device))
    if st not in (0, 8):
        _check("nvfp4pt_workspace_error", st)
    return int(word.value)
