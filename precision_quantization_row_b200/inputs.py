"""Seeded synthetic inputs for the NVFP4 per-token cast (shared by tests and bench).

This module only draws numbers: it holds none of the cast's arithmetic. Every
matrix is drawn in float32 (or float64 where the distribution needs it) with
numpy's PCG64 ``default_rng(seed)`` and rounded once to bfloat16
(round-to-nearest-even, by torch), so the CUDA path and the CPU oracle see the
same bf16 bits.

The shapes and distributions follow the workloads the cast is meant for
(activations with outlier channels, heavy-tailed activations, MoE token groups
aligned to 128 tokens, weights with sparse outliers, and a calibration stream
of activations with a drifting scale).
"""
from __future__ import annotations

import math

import numpy as np
import torch


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """float32/float64 numpy array -> contiguous CPU bfloat16 tensor (RN-even)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


# ------------------------------------------------------------------ configs

def tiny(seed: int = 0, M: int = 256, K: int = 512) -> torch.Tensor:
    """N(0,1) [256, 512]; rows 7 and 100 scaled x40 (outlier tokens); row 3 all zero."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K), dtype=np.float32)
    x[7] *= 40.0
    x[100] *= 40.0
    x[3] = 0.0
    return to_bf16(x)


def dense(seed: int = 1, M: int = 4096, K: int = 4096) -> torch.Tensor:
    """Student-t(3) entries times a per-row lognormal(0, 1) factor: heavy tails
    within rows and a wide spread of row amaxes."""
    rng = np.random.default_rng(seed)
    t = rng.standard_t(3, (M, K))
    s = rng.lognormal(0.0, 1.0, (M, 1))
    return to_bf16(t * s)


def llm(seed: int = 2, M: int = 16384, K: int = 8192, frac: float = 0.01, scale: float = 50.0) -> torch.Tensor:
    """N(0,1) activations with round(1% of K) outlier channels scaled x50."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K), dtype=np.float32)
    n_out = int(round(frac * K))
    cols = rng.choice(K, n_out, replace=False)
    x[:, cols] *= scale
    return to_bf16(x)


def moe_counts(seed: int = 3, experts: int = 64, tokens: int = 65536, align: int = 128) -> np.ndarray:
    """Multinomial token counts per expert, each a multiple of `align`, summing to `tokens`."""
    rng = np.random.default_rng(seed)
    chunks = rng.multinomial(tokens // align, [1.0 / experts] * experts)
    return (chunks * align).astype(np.int64)


def moe(seed: int = 3, experts: int = 64, tokens: int = 65536, K: int = 7168, align: int = 128):
    """(X, offsets): N(0,1) rows scaled by their expert's std ~ U[0.5, 4].
    offsets has experts+1 entries, offsets[0] = 0, offsets[-1] = tokens."""
    rng = np.random.default_rng(seed)
    chunks = rng.multinomial(tokens // align, [1.0 / experts] * experts)
    counts = (chunks * align).astype(np.int64)
    std = rng.uniform(0.5, 4.0, experts).astype(np.float32)
    x = rng.standard_normal((tokens, K), dtype=np.float32)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    for g in range(experts):
        x[offsets[g]:offsets[g + 1]] *= std[g]
    return to_bf16(x), offsets


def weight(seed: int = 4, N: int = 28672, K: int = 8192, outlier_p: float = 0.001, scale: float = 100.0):
    """0.02 * N(0,1) weights; each entry independently (p = 0.1%) scaled x100."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    mask = rng.random((N, K), dtype=np.float32) < outlier_p
    w[mask] *= scale
    return to_bf16(w)


def calib_sigma(t: int) -> float:
    return 1.0 + 0.5 * math.sin(t / 20.0)


def calib_step(t: int, M: int = 8192, K: int = 4096, device: str = "cuda") -> torch.Tensor:
    """Calibration-stream activation t: sigma_t * N(0,1) drawn by a torch generator
    seeded 4000 + t on `device` (drawing on the GPU avoids billions of host normals),
    then rounded to bf16."""
    g = torch.Generator(device=device)
    g.manual_seed(4000 + t)
    a = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    return (a * calib_sigma(t)).to(torch.bfloat16)


def random_shape(seed: int, M: int, K: int, kind: str = "normal") -> torch.Tensor:
    """Generic small inputs for edge-case tests. kind: normal | wide | tiny | zeros | signed_zero."""
    rng = np.random.default_rng(seed)
    if kind == "normal":
        x = rng.standard_normal((M, K), dtype=np.float32)
    elif kind == "wide":  # per-row scales spread over ~60 binades, plus zero blocks
        x = rng.standard_normal((M, K), dtype=np.float32)
        x *= np.exp2(rng.integers(-30, 30, (M, 1))).astype(np.float32)
        x[:, :16] = 0.0
    elif kind == "tiny":  # bf16 subnormal / near-underflow rows
        x = rng.standard_normal((M, K), dtype=np.float32) * np.float32(1e-39)
    elif kind == "zeros":
        x = np.zeros((M, K), np.float32)
    elif kind == "signed_zero":
        x = np.where(rng.random((M, K)) < 0.5, np.float32(-0.0), np.float32(0.0)).astype(np.float32)
    else:
        raise ValueError(kind)
    return to_bf16(x)
