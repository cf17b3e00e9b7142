"""Helpers of the GPU parity tests: run the CUDA path, run the oracle (in parallel
over exact sub-problems for the large workloads), compare element by element.

Sub-problems used for the parallel oracle are exact restrictions of the cast: the
rowwise outputs of a row range depend only on those rows; the columnwise outputs of
a column range only on those columns; each token group's columnwise outputs only on
the group's rows; the 2D weight outputs of a run of 16-row bands only on those rows.
"""
from __future__ import annotations

import concurrent.futures as cf
import multiprocessing as mp
import os
import tempfile

import numpy as np
import torch

import oracle

ROWWISE, COLWISE = 1, 2

# Scratch files of the oracle's worker pool live inside the repository (git-ignored).
_SCRATCH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), ".test_scratch")


def _scratch_dir() -> tempfile.TemporaryDirectory:
    os.makedirs(_SCRATCH, exist_ok=True)
    return tempfile.TemporaryDirectory(dir=_SCRATCH)


def to_np(out: dict) -> dict:
    return {k: v.detach().cpu().numpy() for k, v in out.items()}


def bits_of(x: torch.Tensor) -> np.ndarray:
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def compare(got: dict, want: dict, keys=None, label="") -> None:
    """Bit-exact comparison; floats compared as their bit patterns."""
    keys = keys or sorted(want)
    for k in keys:
        g = np.atleast_1d(np.asarray(got[k]))
        w = np.atleast_1d(np.asarray(want[k], dtype=np.float32 if np.isscalar(want[k]) else None))
        assert g.shape == w.shape or g.size == w.size, (label, k, g.shape, w.shape)
        g = g.reshape(w.shape)
        if w.dtype == np.float32:
            g, w = g.view(np.uint32), w.view(np.uint32)
        bad = np.nonzero(g != w)
        n = bad[0].size
        if n:
            idx = tuple(b[:8] for b in bad)
            raise AssertionError(f"{label} {k}: {n} of {w.size} differ; first at {list(zip(*idx))}: "
                                 f"got {g[idx]} want {w[idx]}")


# ------------------------------------------------------------ parallel oracle

def _worker(task):
    kind, path, a, b, extra = task
    x = np.load(path, mmap_mode="r")
    if kind == "rows":
        return kind, a, b, oracle.quantize(np.ascontiguousarray(x[a:b]), flags=ROWWISE)
    if kind == "cols":
        return kind, a, b, oracle.quantize(np.ascontiguousarray(x[:, a:b]), flags=COLWISE)
    if kind == "group":
        return kind, a, b, oracle.quantize(np.ascontiguousarray(x[a:b]), flags=COLWISE)
    if kind == "w2d":
        return kind, a, b, oracle.quantize_weight_2d(np.ascontiguousarray(x[a:b]))
    if kind == "colopts":
        return kind, a, b, oracle.quantize_colwise_opts(np.ascontiguousarray(x[:, a:b]), col_base=a, **extra)
    raise ValueError(kind)


def _pool(n_tasks):
    workers = max(1, min(n_tasks, os.cpu_count() or 1, 32))
    return cf.ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn"))


def _split(n, parts, align=16):
    step = max(align, -(-n // parts) // align * align)
    return [(a, min(n, a + step)) for a in range(0, n, step)]


def oracle_quantize_parallel(x: torch.Tensor, flags=ROWWISE | COLWISE, offsets=None, parts=None) -> dict:
    """The oracle's cast of x, computed over exact sub-problems in a spawn pool."""
    xb = bits_of(x)
    M, K = xb.shape
    parts = parts or max(1, min(32, os.cpu_count() or 1)) * 2
    out = {"amax_row": np.zeros(M, np.float32)}
    with _scratch_dir() as d:
        path = os.path.join(d, "x.npy")
        np.save(path, xb)
        tasks = [("rows", path, a, b, None) for a, b in _split(M, parts)]
        if flags & ROWWISE:
            out["q_row"] = np.zeros((M, K // 2), np.uint8)
            out["sf_row"] = np.zeros((M, K // 16), np.uint8)
        if flags & COLWISE:
            if offsets is None:
                out["q_col"] = np.zeros((K, M // 2), np.uint8)
                out["sf_col"] = np.zeros((K, M // 16), np.uint8)
                out["amax_col"] = np.zeros(K, np.float32)
                tasks += [("cols", path, a, b, None) for a, b in _split(K, parts)]
            else:
                G = len(offsets) - 1
                out["q_col"] = np.zeros(K * M // 2, np.uint8)
                out["sf_col"] = np.zeros(K * M // 16, np.uint8)
                out["amax_col"] = np.zeros((G, K), np.float32)
                tasks += [("group", path, int(offsets[g]), int(offsets[g + 1]), g)
                          for g in range(G) if offsets[g + 1] > offsets[g]]
        with _pool(len(tasks)) as ex:
            futs = {ex.submit(_worker, t): t for t in tasks}
            for f in cf.as_completed(futs):
                kind, a, b, r = f.result()
                g = futs[f][4]
                if kind == "rows":
                    out["amax_row"][a:b] = r["amax_row"]
                    if flags & ROWWISE:
                        out["q_row"][a:b] = r["q_row"]
                        out["sf_row"][a:b] = r["sf_row"]
                elif kind == "cols":
                    out["q_col"][a:b] = r["q_col"]
                    out["sf_col"][a:b] = r["sf_col"]
                    out["amax_col"][a:b] = r["amax_col"]
                else:  # group
                    out["q_col"][K * a // 2:K * b // 2] = r["q_col"].ravel()
                    out["sf_col"][K * a // 16:K * b // 16] = r["sf_col"].ravel()
                    out["amax_col"][g] = r["amax_col"]
    if not flags & ROWWISE:
        out.pop("amax_row")
    return out


def oracle_colwise_opts_parallel(x: torch.Tensor, offsets=None, parts=None, **opts) -> dict:
    """The oracle's columnwise cast with the options (rht, rht_signs, sr, seed, offset) over
    column ranges in a spawn pool: a column's outputs depend on that column alone (the
    random words take its index in the full matrix). Outputs shaped as
    oracle.quantize_colwise_opts's."""
    xb = bits_of(x)
    M, K = xb.shape
    parts = parts or max(1, min(32, os.cpu_count() or 1)) * 2
    G = 1 if offsets is None else len(offsets) - 1
    off = [0, M] if offsets is None else [int(o) for o in offsets]
    q = np.zeros(K * M // 2, np.uint8)
    sf = np.zeros(K * M // 16, np.uint8)
    am = np.zeros((G, K), np.float32)
    with _scratch_dir() as d:
        path = os.path.join(d, "x.npy")
        np.save(path, xb)
        tasks = [("colopts", path, a, b, dict(opts, offsets=off)) for a, b in _split(K, parts)]
        with _pool(len(tasks)) as ex:
            for kind, a, b, r in ex.map(_worker, tasks):
                am[:, a:b] = r["amax_col"]
                for g in range(G):
                    r0, m = off[g], off[g + 1] - off[g]
                    qg = r["q_col"][(b - a) * r0 // 2:(b - a) * (r0 + m) // 2].reshape(b - a, m // 2)
                    sg = r["sf_col"][(b - a) * r0 // 16:(b - a) * (r0 + m) // 16].reshape(b - a, m // 16)
                    q[K * r0 // 2 + a * (m // 2):K * r0 // 2 + b * (m // 2)] = qg.ravel()
                    sf[K * r0 // 16 + a * (m // 16):K * r0 // 16 + b * (m // 16)] = sg.ravel()
    if offsets is None:
        return {"q_col": q.reshape(K, M // 2), "sf_col": sf.reshape(K, M // 16), "amax_col": am.reshape(K)}
    return {"q_col": q, "sf_col": sf, "amax_col": am}


def oracle_weight_2d_parallel(w: torch.Tensor, parts=None) -> dict:
    wb = bits_of(w)
    N, K = wb.shape
    parts = parts or max(1, min(32, os.cpu_count() or 1)) * 2
    out = {"q_row": np.zeros((N, K // 2), np.uint8), "sf_row": np.zeros((N, K // 16), np.uint8),
           "amax_row": np.zeros(N, np.float32)}
    with _scratch_dir() as d:
        path = os.path.join(d, "w.npy")
        np.save(path, wb)
        tasks = [("w2d", path, a, b, None) for a, b in _split(N, parts)]
        with _pool(len(tasks)) as ex:
            for kind, a, b, r in ex.map(_worker, tasks):
                for k in out:
                    out[k][a:b] = r[k]
    return out


# Canary bytes around device buffers: the stand-in for a memory sanitizer (none runs on
# the GPU pool). Each buffer sits inside a larger uint8 allocation with GUARD bytes of
# CANARY on each side; a write outside the buffer changes one of them.
GUARD = 256      # bytes on each side; keeps the buffer 256-byte aligned
CANARY = 0xA5


def guarded(shape, dtype, device) -> tuple:
    """(raw, view): `view` is a contiguous `dtype` tensor of `shape` inside `raw`."""
    n = int(np.prod(shape, dtype=np.int64)) * torch.empty((), dtype=dtype).element_size()
    raw = torch.full((2 * GUARD + n,), CANARY, dtype=torch.uint8, device=device)
    return raw, raw[GUARD:GUARD + n].view(dtype).view(tuple(shape))


def canaries_intact(raw: torch.Tensor) -> bool:
    r = raw.detach().cpu()
    return bool((r[:GUARD] == CANARY).all()) and bool((r[-GUARD:] == CANARY).all())


def guarded_outputs(rows: int, cols: int, flags: int, device, groups: int = 1) -> tuple:
    """([raw, ...], out): the cast's output dict (the binding's shapes) in guarded buffers."""
    shapes = {}
    if flags & ROWWISE:
        shapes.update(q_row=((rows, cols // 2), torch.uint8), sf_row=((rows, cols // 16), torch.uint8),
                      amax_row=((rows,), torch.float32))
    if flags & COLWISE:
        if groups == 1:
            shapes.update(q_col=((cols, rows // 2), torch.uint8), sf_col=((cols, rows // 16), torch.uint8),
                          amax_col=((cols,), torch.float32))
        else:
            shapes.update(q_col=((cols * rows // 2,), torch.uint8), sf_col=((cols * rows // 16,), torch.uint8),
                          amax_col=((groups, cols), torch.float32))
    raws, out = [], {}
    for k, (shape, dtype) in shapes.items():
        raw, out[k] = guarded(shape, dtype, device)
        raws.append(raw)
    return raws, out
