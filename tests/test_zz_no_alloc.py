"""nvfp4pt_quantize_grouped_noalloc against nvfp4pt_quantize_grouped, through the C ABI.

The no-allocation entry point serves callers that must not allocate device memory
themselves (code running inside an allocator or memory-pool callback, under a fixed
memory budget, or without a workspace to pass); its scratch lives in a static device
array inside the library. It must give the same bits as the workspace entry point, on
consecutive calls too (the shared array keeps the previous call's contents, which each
call clears before use), and must refuse token-group counts its array cannot hold.

This file is collected last on purpose, so a run that stops at the first failure has
run every other test first; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import precision_quantization_row_b200 as nv
from precision_quantization_row_b200 import inputs

pytestmark = pytest.mark.gpu

NOALLOC_MAX_GROUPS = 252  # NVFP4PT_NOALLOC_MAX_GROUPS in include/nvfp4pt.h


def _outputs(rows, cols, G):
    return {
        "q_row": torch.full((rows, cols // 2), 0xA5, dtype=torch.uint8, device="cuda"),
        "sf_row": torch.full((rows, cols // 16), 0xA5, dtype=torch.uint8, device="cuda"),
        "amax_row": torch.full((rows,), -1.0, dtype=torch.float32, device="cuda"),
        "q_col": torch.full((cols * rows // 2,), 0xA5, dtype=torch.uint8, device="cuda"),
        "sf_col": torch.full((cols * rows // 16,), 0xA5, dtype=torch.uint8, device="cuda"),
        "amax_col": torch.full((G, cols), -1.0, dtype=torch.float32, device="cuda"),
        "absmax": torch.full((G,), 3.0, dtype=torch.float32, device="cuda"),
    }


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _call(noalloc: bool, x, offsets, out, decay=0.5):
    L = nv.lib()
    rows, cols = x.shape
    G = len(offsets) - 1
    off = (ctypes.c_int64 * len(offsets))(*[int(o) for o in offsets])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = [_p(x), rows, cols, off, G, nv.ROWWISE | nv.COLWISE, _p(out["q_row"]), _p(out["sf_row"]),
            _p(out["amax_row"]), _p(out["q_col"]), _p(out["sf_col"]), _p(out["amax_col"]), _p(out["absmax"]),
            ctypes.c_float(decay)]
    if noalloc:
        return L.nvfp4pt_quantize_grouped_noalloc(*args, stream)
    ws = torch.empty(nv.workspace_bytes(rows, cols, G), dtype=torch.uint8, device="cuda")
    return L.nvfp4pt_quantize_grouped(*args, _p(ws), stream)


def _same(a, b, label):
    for k in a:
        x = a[k].cpu().numpy()
        y = b[k].cpu().numpy()
        if x.dtype == np.float32:
            x, y = x.view(np.uint32), y.view(np.uint32)
        assert np.array_equal(x, y), f"{label}: {k} differs"


def test_noalloc_matches_workspace_entry_on_consecutive_calls():
    cases = [
        (inputs.random_shape(21, 400, 272, "wide"), [0, 16, 48, 48, 400]),
        (inputs.random_shape(22, 1040, 1056, "normal"), [0, 128, 512, 512, 1040]),
    ]
    for i, (x, offsets) in enumerate(cases):
        xd = x.cuda()
        G = len(offsets) - 1
        ref = _outputs(*x.shape, G)
        got = _outputs(*x.shape, G)
        assert _call(False, xd, offsets, ref) == 0
        assert _call(True, xd, offsets, got) == 0
        torch.cuda.synchronize()
        _same(ref, got, f"call {i}")


def test_noalloc_refuses_more_groups_than_its_scratch_holds():
    rows, cols = 16 * (NOALLOC_MAX_GROUPS + 1), 16
    x = torch.zeros((rows, cols), dtype=torch.bfloat16, device="cuda")
    offsets = list(range(0, rows + 1, 16))
    out = _outputs(rows, cols, NOALLOC_MAX_GROUPS + 1)
    assert _call(True, x, offsets, out) == 4  # NVFP4PT_ERR_GROUPS, nothing launched
    assert (out["amax_row"] == -1.0).all()
    ok = offsets[:NOALLOC_MAX_GROUPS] + [rows]  # the largest count that fits
    out = _outputs(rows, cols, NOALLOC_MAX_GROUPS)
    ref = _outputs(rows, cols, NOALLOC_MAX_GROUPS)
    assert _call(True, x, ok, out) == 0
    assert _call(False, x, ok, ref) == 0
    torch.cuda.synchronize()
    _same(ref, out, "252 groups")
