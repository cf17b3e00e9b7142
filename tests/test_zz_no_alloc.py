"""nvfp4pt_quantize_grouped_noalloc through the C ABI: against nvfp4pt_quantize_grouped
and against the oracle.

The no-allocation entry point serves callers that must not allocate device memory
themselves (code running inside an allocator or memory-pool callback, under a fixed
memory budget, or without a workspace to pass); its scratch lives in a static device
array inside the library. It must give the same bits as the workspace entry point and
as the oracle, on consecutive calls too: the shared array keeps the previous call's
contents, which each call clears before use, so a call with large group maxima is
followed by one with small maxima on the same groups. It must refuse token-group
counts its array cannot hold.

This file is collected last on purpose, so a run that stops at the first failure has
run every other test first; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import precision_quantization_row_b200 as nv
from precision_quantization_row_b200 import inputs
from parity_util import compare, oracle_quantize_parallel, to_np

pytestmark = pytest.mark.gpu

NOALLOC_MAX_GROUPS = 252  # NVFP4PT_NOALLOC_MAX_GROUPS in include/nvfp4pt.h
RC = nv.ROWWISE | nv.COLWISE


def _outputs(rows, cols, G, flags=RC, absmax=True):
    out = {}
    if flags & nv.ROWWISE:
        out["q_row"] = torch.full((rows, cols // 2), 0xA5, dtype=torch.uint8, device="cuda")
        out["sf_row"] = torch.full((rows, cols // 16), 0xA5, dtype=torch.uint8, device="cuda")
        out["amax_row"] = torch.full((rows,), -1.0, dtype=torch.float32, device="cuda")
    if flags & nv.COLWISE:
        out["q_col"] = torch.full((cols * rows // 2,), 0xA5, dtype=torch.uint8, device="cuda")
        out["sf_col"] = torch.full((cols * rows // 16,), 0xA5, dtype=torch.uint8, device="cuda")
        out["amax_col"] = torch.full((G, cols), -1.0, dtype=torch.float32, device="cuda")
    if absmax:
        out["absmax"] = torch.full((G,), 3.0, dtype=torch.float32, device="cuda")
    return out


def _p(t):
    return ctypes.c_void_p(None if t is None else t.data_ptr())


def _call(noalloc: bool, x, offsets, out, flags=RC, decay=0.5):
    L = nv.lib()
    rows, cols = x.shape
    G = len(offsets) - 1
    off = (ctypes.c_int64 * len(offsets))(*[int(o) for o in offsets])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = [_p(x), rows, cols, off, G, flags, _p(out.get("q_row")), _p(out.get("sf_row")), _p(out.get("amax_row")),
            _p(out.get("q_col")), _p(out.get("sf_col")), _p(out.get("amax_col")), _p(out.get("absmax")),
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


def _want(orc, x, offsets, flags=RC, absmax=True, decay=0.5):
    G = len(offsets) - 1
    bufs = np.full(G, 3.0, np.float32) if absmax else None
    return orc.quantize_grouped(x, offsets, flags=flags, absmax=bufs, decay=decay)


# (x, offsets): the row pass (two widths), empty and ragged groups, and rows wider than
# 16384 elements (the tile path)
CASES = {
    "400x272": (lambda: inputs.random_shape(21, 400, 272, "wide"), [0, 16, 48, 48, 400]),
    "1040x1056": (lambda: inputs.random_shape(22, 1040, 1056, "normal"), [0, 128, 512, 512, 1040]),
    "128x16400_tile_path": (lambda: inputs.random_shape(23, 128, 16400, "wide"), [0, 48, 48, 112, 128]),
}


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_workspace_entry_and_oracle_on_consecutive_calls(orc, name):
    """Two calls in a row on the same groups: first on 100 x (large group maxima left in
    the shared array), then on x. Both against the workspace entry; the second also
    against the oracle."""
    make, offsets = CASES[name]
    x = make()
    G = len(offsets) - 1
    xd = x.cuda()
    for i, xi in enumerate((xd * 100, xd)):
        ref = _outputs(*x.shape, G)
        got = _outputs(*x.shape, G)
        assert _call(False, xi, offsets, ref) == 0
        assert _call(True, xi, offsets, got) == 0
        torch.cuda.synchronize()
        _same(ref, got, f"{name} call {i}")
    compare(to_np(got), _want(orc, x, offsets), label=f"{name} vs oracle")


def test_noalloc_colwise_only_without_buffers(orc):
    """Columnwise outputs alone, no running buffers (absmax NULL), after a row+column
    call with buffers on larger values."""
    x = inputs.random_shape(24, 272, 144, "normal")
    offsets = [0, 144, 160, 272]
    G = len(offsets) - 1
    xd = x.cuda()
    assert _call(True, xd * 64, offsets, _outputs(272, 144, G)) == 0
    got = _outputs(272, 144, G, flags=nv.COLWISE, absmax=False)
    ref = _outputs(272, 144, G, flags=nv.COLWISE, absmax=False)
    assert _call(True, xd, offsets, got, flags=nv.COLWISE) == 0
    assert _call(False, xd, offsets, ref, flags=nv.COLWISE) == 0
    torch.cuda.synchronize()
    _same(ref, got, "colwise only")
    want = _want(orc, x, offsets, flags=nv.COLWISE, absmax=False)
    want.pop("amax_row")   # the oracle reports it always; the call was not asked for it
    compare(to_np(got), want, label="colwise only vs oracle")


def test_noalloc_most_groups_vs_oracle(orc):
    """252 token groups (the most the static array holds), many of them empty."""
    rng = np.random.default_rng(25)
    G = NOALLOC_MAX_GROUPS
    sizes = rng.multinomial(160, [1 / G] * G) * 16
    offsets = np.concatenate([[0], np.cumsum(sizes)]).tolist()
    x = inputs.random_shape(26, offsets[-1], 64, "wide")
    got = _outputs(offsets[-1], 64, G)
    assert _call(True, x.cuda(), offsets, got) == 0
    torch.cuda.synchronize()
    compare(to_np(got), _want(orc, x, offsets), label="252 groups vs oracle")


@pytest.mark.slow
def test_noalloc_moe_config_full_vs_oracle(orc):
    """The MoE workload (65536 x 7168, 64 token groups) through the entry without
    allocation, element by element against the oracle."""
    x, offsets = inputs.moe()
    G = len(offsets) - 1
    got = _outputs(*x.shape, G)
    got["absmax"].fill_(1.0)
    assert _call(True, x.cuda(), offsets, got, decay=0.5) == 0
    torch.cuda.synchronize()
    got = to_np(got)
    want = oracle_quantize_parallel(x, offsets=offsets)
    want["amax_col"] = want["amax_col"].reshape(G, -1)
    compare({k: v for k, v in got.items() if k != "absmax"}, want, label="moe noalloc")
    obs = np.array([want["amax_col"][g].max() for g in range(G)], np.float32)
    assert np.array_equal(got["absmax"], np.maximum(np.float32(0.5), obs))


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
