"""ctypes front-end of the plain C oracle of the NVFP4 per-token cast.

TEST INFRASTRUCTURE ONLY: the test-suite, the smoke check and the benchmark's
CPU-baseline leg are its only users. The CUDA library never imports or links
it, and it shares no code with the CUDA path.

All arrays here are host numpy arrays; bf16 inputs travel as their uint16 bit
patterns. See nvfp4pt_oracle.c for the definition, its sources and readings.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4pt_oracle.c")
_LIB = os.path.join(_HERE, "libnvfp4pt_oracle.so")

# IEEE binary32 arithmetic, one rounding per operation: no FMA contraction,
# no fast-math, no flush-to-zero.
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fno-unsafe-math-optimizations",
          "-std=c11", "-shared", "-fPIC", "-Wall", "-Wextra"]

ROWWISE = 1
COLWISE = 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (if missing or older than its source)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        F = ctypes.c_float
        U8 = ctypes.c_uint8
        _lib.oracle_e4m3.argtypes, _lib.oracle_e4m3.restype = [F], U8
        _lib.oracle_e2m1.argtypes, _lib.oracle_e2m1.restype = [F], U8
        _lib.oracle_e4m3_decode.argtypes, _lib.oracle_e4m3_decode.restype = [U8], F
        _lib.oracle_e2m1_decode.argtypes, _lib.oracle_e2m1_decode.restype = [U8], F
        _lib.oracle_bf16_to_f32.argtypes, _lib.oracle_bf16_to_f32.restype = [ctypes.c_uint16], F
        _lib.oracle_s_enc.argtypes, _lib.oracle_s_enc.restype = [F], F
        _lib.oracle_block_scale_arg.argtypes, _lib.oracle_block_scale_arg.restype = [F, F], F
        _lib.oracle_block_enc.argtypes, _lib.oracle_block_enc.restype = [U8, F], F
        _lib.oracle_amax_rows.argtypes, _lib.oracle_amax_rows.restype = [P, I64, I64, P], None
        _lib.oracle_amax_cols.argtypes, _lib.oracle_amax_cols.restype = [P, I64, I64, I64, P], None
        _lib.oracle_update_absmax.argtypes = [P, P, I64, F]
        _lib.oracle_update_absmax.restype = None
        _lib.oracle_quantize.argtypes = [P, I64, I64, ctypes.c_int, P, P, P, P, P, P, P, F]
        _lib.oracle_quantize.restype = ctypes.c_int
        _lib.oracle_quantize_grouped.argtypes = [P, I64, I64, P, ctypes.c_int, ctypes.c_int,
                                                 P, P, P, P, P, P, P, F]
        _lib.oracle_quantize_grouped.restype = ctypes.c_int
        _lib.oracle_quantize_weight_2d.argtypes = [P, I64, I64, P, P, P]
        _lib.oracle_quantize_weight_2d.restype = ctypes.c_int
        _lib.oracle_e4m3_array.argtypes, _lib.oracle_e4m3_array.restype = [P, I64, P], None
        _lib.oracle_e2m1_array.argtypes, _lib.oracle_e2m1_array.restype = [P, I64, P], None
        _lib.oracle_f32_to_bf16_array.argtypes, _lib.oracle_f32_to_bf16_array.restype = [P, I64, P], None
        _lib.oracle_dequantize_rows.argtypes = [P, P, P, I64, I64, P]
        _lib.oracle_dequantize_rows.restype = ctypes.c_int
        _lib.oracle_gemm_per_token.argtypes = [P, P, P, I64, P, P, P, I64, I64, P, P]
        _lib.oracle_gemm_per_token.restype = ctypes.c_int
        U32, U64 = ctypes.c_uint32, ctypes.c_uint64
        _lib.oracle_philox4x32_10.argtypes, _lib.oracle_philox4x32_10.restype = [P, P, P], None
        _lib.oracle_sr_word.argtypes, _lib.oracle_sr_word.restype = [I64, I64, U64, U64], U32
        _lib.oracle_rht16.argtypes, _lib.oracle_rht16.restype = [P, U32, P], None
        _lib.oracle_e2m1_sr.argtypes, _lib.oracle_e2m1_sr.restype = [F, U32], U8
        _lib.oracle_quantize_colwise_opts.argtypes = [P, I64, I64, I64, P, ctypes.c_int, ctypes.c_int, U32,
                                                      ctypes.c_int, U64, U64, P, P, P]
        _lib.oracle_quantize_colwise_opts.restype = ctypes.c_int
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bits(x) -> np.ndarray:
    """bf16 input as a C-contiguous uint16 array of bit patterns."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16
            return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x)
    assert x.dtype == np.uint16, "pass bf16 as a torch tensor or as uint16 bit patterns"
    return np.ascontiguousarray(x)


# ----------------------------------------------------------------- scalars

def e4m3(v: float) -> int:
    return int(lib().oracle_e4m3(v))


def e2m1(y: float) -> int:
    return int(lib().oracle_e2m1(y))


def e4m3_decode(code: int) -> float:
    return float(lib().oracle_e4m3_decode(code))


def e2m1_decode(code: int) -> float:
    return float(lib().oracle_e2m1_decode(code))


def s_enc(amax: float) -> float:
    return float(lib().oracle_s_enc(amax))


def block_scale_arg(block_amax: float, s: float) -> float:
    return float(lib().oracle_block_scale_arg(block_amax, s))


def block_enc(sf: int, s: float) -> float:
    return float(lib().oracle_block_enc(sf, s))


# ------------------------------------------------------------------ arrays

def e4m3_array(v) -> np.ndarray:
    v = np.ascontiguousarray(np.asarray(v, np.float32))
    out = np.empty(v.shape, np.uint8)
    lib().oracle_e4m3_array(_ptr(v), v.size, _ptr(out))
    return out


def e2m1_array(y) -> np.ndarray:
    y = np.ascontiguousarray(np.asarray(y, np.float32))
    out = np.empty(y.shape, np.uint8)
    lib().oracle_e2m1_array(_ptr(y), y.size, _ptr(out))
    return out


def amax_rows(x) -> np.ndarray:
    xb = _bits(x)
    M, K = xb.shape
    out = np.empty(M, np.float32)
    lib().oracle_amax_rows(_ptr(xb), M, K, _ptr(out))
    return out


def amax_cols(x, r0: int = 0, r1: int | None = None) -> np.ndarray:
    xb = _bits(x)
    M, K = xb.shape
    r1 = M if r1 is None else r1
    out = np.empty(K, np.float32)
    lib().oracle_amax_cols(_ptr(xb), K, r0, r1, _ptr(out))
    return out


def update_absmax(buf: float, amax_vec, decay: float) -> float:
    b = np.array([buf], np.float32)
    v = np.ascontiguousarray(np.asarray(amax_vec, np.float32))
    lib().oracle_update_absmax(_ptr(b), _ptr(v), v.size, decay)
    return float(b[0])


def quantize(x, flags: int = ROWWISE | COLWISE, absmax: float | None = None, decay: float = 0.0):
    """Per-token cast. Returns a dict of numpy arrays (and 'absmax' if given)."""
    xb = _bits(x)
    M, K = xb.shape
    out = {"amax_row": np.zeros(M, np.float32)}
    if flags & ROWWISE:
        out["q_row"] = np.zeros((M, K // 2), np.uint8)
        out["sf_row"] = np.zeros((M, K // 16), np.uint8)
    if flags & COLWISE:
        out["q_col"] = np.zeros((K, M // 2), np.uint8)
        out["sf_col"] = np.zeros((K, M // 16), np.uint8)
        out["amax_col"] = np.zeros(K, np.float32)
    buf = None if absmax is None else np.array([absmax], np.float32)
    rc = lib().oracle_quantize(_ptr(xb), M, K, flags, _ptr(out.get("q_row")), _ptr(out.get("sf_row")),
                               _ptr(out["amax_row"]), _ptr(out.get("q_col")), _ptr(out.get("sf_col")),
                               _ptr(out.get("amax_col")), _ptr(buf), decay)
    if rc != 0:
        raise ValueError(f"oracle_quantize: bad shape {M}x{K}")
    if buf is not None:
        out["absmax"] = float(buf[0])
    return out


def quantize_grouped(x, offsets, flags: int = ROWWISE | COLWISE, absmax=None, decay: float = 0.0):
    """Grouped cast. offsets: G+1 row offsets. Column outputs are flat byte arrays
    (group g's [K, m_g/2] block starts at K*offsets[g]/2)."""
    xb = _bits(x)
    M, K = xb.shape
    off = np.ascontiguousarray(np.asarray(offsets, np.int64))
    G = off.size - 1
    out = {"amax_row": np.zeros(M, np.float32)}
    if flags & ROWWISE:
        out["q_row"] = np.zeros((M, K // 2), np.uint8)
        out["sf_row"] = np.zeros((M, K // 16), np.uint8)
    if flags & COLWISE:
        out["q_col"] = np.zeros(K * M // 2, np.uint8)
        out["sf_col"] = np.zeros(K * M // 16, np.uint8)
        out["amax_col"] = np.zeros((G, K), np.float32)
    bufs = None if absmax is None else np.ascontiguousarray(np.asarray(absmax, np.float32)).copy()
    rc = lib().oracle_quantize_grouped(_ptr(xb), M, K, _ptr(off), G, flags, _ptr(out.get("q_row")),
                                       _ptr(out.get("sf_row")), _ptr(out["amax_row"]),
                                       _ptr(out.get("q_col")), _ptr(out.get("sf_col")),
                                       _ptr(out.get("amax_col")), _ptr(bufs), decay)
    if rc != 0:
        raise ValueError("oracle_quantize_grouped: bad shape or offsets")
    if bufs is not None:
        out["absmax"] = bufs
    return out


def quantize_weight_2d(w):
    wb = _bits(w)
    N, K = wb.shape
    out = {"q_row": np.zeros((N, K // 2), np.uint8), "sf_row": np.zeros((N, K // 16), np.uint8),
           "amax_row": np.zeros(N, np.float32)}
    rc = lib().oracle_quantize_weight_2d(_ptr(wb), N, K, _ptr(out["q_row"]), _ptr(out["sf_row"]),
                                         _ptr(out["amax_row"]))
    if rc != 0:
        raise ValueError(f"oracle_quantize_weight_2d: bad shape {N}x{K}")
    return out


def dequantize_rows(q, sf, amax):
    """Reconstruct x ~ val(q) * float(sf) / s_enc (rowwise layout), in float64.
    Used only by the round-trip bound tests."""
    q = np.asarray(q, np.uint8)
    M, half = q.shape
    K = half * 2
    lo = q & 0xF
    hi = q >> 4
    codes = np.empty((M, K), np.uint8)
    codes[:, 0::2] = lo
    codes[:, 1::2] = hi
    table = np.array([e2m1_decode(c) for c in range(16)], np.float64)
    sft = np.array([e4m3_decode(c) if c != 0x7F and c != 0xFF else np.nan for c in range(256)], np.float64)
    vals = table[codes]
    scale = sft[np.asarray(sf, np.uint8)].repeat(16, axis=1)
    senc = np.array([s_enc(float(a)) for a in np.asarray(amax, np.float32)], np.float64)[:, None]
    return vals * scale / senc


def f32_to_bf16(v) -> np.ndarray:
    """uint16 bits of the nearest bf16 to each binary32 value (ties to even)."""
    a = np.ascontiguousarray(np.asarray(v, np.float32))
    out = np.zeros(a.shape, np.uint16)
    lib().oracle_f32_to_bf16_array(_ptr(a), a.size, _ptr(out))
    return out


def dequantize(q, sf, amax) -> np.ndarray:
    """oracle_dequantize_rows: bf16 bits [M, K] of rowwise-layout NVFP4 data
    (q [M, K/2], sf [M, K/16], amax [M]); columnwise data [K, M/2], [K, M/16], [K]
    give X^T."""
    qa = np.ascontiguousarray(np.asarray(q, np.uint8))
    M, half = qa.shape
    K = 2 * half
    sfa = np.ascontiguousarray(np.asarray(sf, np.uint8).reshape(M, K // 16))
    am = np.ascontiguousarray(np.asarray(amax, np.float32).reshape(M))
    out = np.zeros((M, K), np.uint16)
    if lib().oracle_dequantize_rows(_ptr(qa), _ptr(sfa), _ptr(am), M, K, _ptr(out)) != 0:
        raise ValueError(f"oracle_dequantize_rows: bad shape {M}x{K}")
    return out


def requantize_colwise(q_row, sf_row, amax_row, offsets=None, absmax=None, decay: float = 0.0) -> dict:
    """Columnwise requantization of rowwise-quantized data: the columnwise cast (per
    token group when offsets are given) of X' = dequantize(q_row, sf_row, amax_row),
    the NVFP4 per-token analog of the "dequantize, then columnwise-only requantize"
    step of TransformerEngine PR #3244 (flowchart). It adds no arithmetic of its own:
    both steps are the oracle's dequantize and cast."""
    xd = dequantize(q_row, sf_row, amax_row)
    M = xd.shape[0]
    off = [0, M] if offsets is None else offsets
    out = quantize_grouped(xd.view(np.uint16), off, flags=COLWISE, absmax=absmax, decay=decay)
    res = {k: out[k] for k in ("q_col", "sf_col", "amax_col")}
    if offsets is None:
        res["q_col"] = res["q_col"].reshape(xd.shape[1], M // 2)
        res["sf_col"] = res["sf_col"].reshape(xd.shape[1], M // 16)
        res["amax_col"] = res["amax_col"].reshape(-1)
    if "absmax" in out:
        res["absmax"] = out["absmax"]
    return res


def gemm_per_token(qa, sfa, amax_a, qb, sfb, amax_b):
    """oracle_gemm_per_token: D [M, N] (float64) of two K-major rowwise-layout NVFP4
    operands (A: q [M, K/2], sf [M, K/16], amax [M]; B: q [N, K/2], sf [N, K/16],
    amax [N]), D = S_dec(amax_a) S_dec(amax_b) * sum_k val*sf*val*sf with the sum
    exact; also the same expression over the terms' magnitudes, [M, N]."""
    qa = np.ascontiguousarray(np.asarray(qa, np.uint8))
    qb = np.ascontiguousarray(np.asarray(qb, np.uint8))
    M, half = qa.shape
    N = qb.shape[0]
    K = 2 * half
    if qb.shape[1] != half:
        raise ValueError("operands differ in K")
    sa = np.ascontiguousarray(np.asarray(sfa, np.uint8).reshape(M, K // 16))
    sb = np.ascontiguousarray(np.asarray(sfb, np.uint8).reshape(N, K // 16))
    aa = np.ascontiguousarray(np.asarray(amax_a, np.float32).reshape(M))
    ab = np.ascontiguousarray(np.asarray(amax_b, np.float32).reshape(N))
    out = np.zeros((M, N), np.float64)
    mag = np.zeros((M, N), np.float64)
    st = lib().oracle_gemm_per_token(_ptr(qa), _ptr(sa), _ptr(aa), M, _ptr(qb), _ptr(sb), _ptr(ab), N, K,
                                     _ptr(out), _ptr(mag))
    if st == -1:
        raise ValueError(f"oracle_gemm_per_token: bad shape M={M} N={N} K={K}")
    if st == -2:
        raise ValueError("oracle_gemm_per_token: a block scale is not a non-negative finite e4m3fn code")
    return out, mag


# ------------------------------------------- columnwise options: RHT and SR

def philox4x32_10(ctr, key) -> np.ndarray:
    """oracle_philox4x32_10: four 32-bit words of Philox4x32-10 at counter ctr (4 words)
    with key (2 words)."""
    c = np.ascontiguousarray(np.asarray(ctr, np.uint32))
    k = np.ascontiguousarray(np.asarray(key, np.uint32))
    out = np.zeros(4, np.uint32)
    lib().oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def sr_word(m: int, k: int, seed: int, offset: int) -> int:
    """The random word of columnwise element (row m, column k)."""
    return int(lib().oracle_sr_word(m, k, seed, offset))


def rht16(v, signs: int) -> np.ndarray:
    """(1/4) H16 S v by the four binary32 butterfly stages."""
    a = np.ascontiguousarray(np.asarray(v, np.float32).reshape(16))
    out = np.zeros(16, np.float32)
    lib().oracle_rht16(_ptr(a), signs, _ptr(out))
    return out


def e2m1_sr(y: float, r: int) -> int:
    return int(lib().oracle_e2m1_sr(y, r))


def quantize_colwise_opts(x, offsets=None, rht: bool = False, rht_signs: int = 0, sr: bool = False,
                          seed: int = 0, offset: int = 0, col_base: int = 0) -> dict:
    """The columnwise direction with the RHT / SR options. offsets None: one group, and
    the outputs are shaped as quantize's ([K, M/2], [K, M/16], [K]); else as
    quantize_grouped's (flat codes and scales, amax_col [G, K]). col_base: the column
    index of x's first column in the full matrix (for the random words)."""
    xb = _bits(x)
    M, K = xb.shape
    off = np.ascontiguousarray(np.asarray([0, M] if offsets is None else offsets, np.int64))
    G = off.size - 1
    q = np.zeros(K * M // 2, np.uint8)
    sf = np.zeros(K * M // 16, np.uint8)
    am = np.zeros((G, K), np.float32)
    rc = lib().oracle_quantize_colwise_opts(_ptr(xb), M, K, col_base, _ptr(off), G, int(rht), rht_signs & 0xFFFF,
                                            int(sr),
                                            seed, offset, _ptr(q), _ptr(sf), _ptr(am))
    if rc != 0:
        raise ValueError("oracle_quantize_colwise_opts: bad shape or offsets")
    if offsets is None:
        return {"q_col": q.reshape(K, M // 2), "sf_col": sf.reshape(K, M // 16), "amax_col": am.reshape(K)}
    return {"q_col": q, "sf_col": sf, "amax_col": am}
