"""A second, independent restatement of the cast in exact rationals, against the C oracle.

This is a cross-check of the C code (operation order, rounding of each binary32 step,
clamps, layouts), written in another language with exact arithmetic: each binary32
operation is computed exactly as a Fraction and then rounded to nearest-even binary32
(with subnormals and overflow to infinity). It restates the same definition, so it
does not replace the pins in the other oracle tests; it catches slips in the C.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from precision_quantization_row_b200 import inputs

FLT_MAX = Fraction((1 << 24) - 1) * Fraction(2) ** 104
INF = None  # sentinel for binary32 overflow


def rn32(q: Fraction):
    """Round a rational to the nearest binary32 (ties to even); None on overflow."""
    if q == 0:
        return Fraction(0)
    neg = q < 0
    a = -q if neg else q
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    quantum = Fraction(2) ** (max(e, -126) - 23)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    r = fl * quantum
    if r > FLT_MAX:
        return INF
    return -r if neg else r


E2M1 = [Fraction(v) for v in ("0", "1/2", "1", "3/2", "2", "3", "4", "6")]


def e4m3_values():
    vals = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        vals.append(Fraction(m, 8) * Fraction(2) ** -6 if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7))
    return vals


E4M3 = e4m3_values()


def nearest_even(a: Fraction, table, cap_code):
    if a > table[cap_code]:
        return cap_code
    best, bd = 0, None
    for c, v in enumerate(table):
        d = abs(v - a)
        if bd is None or d < bd or (d == bd and c % 2 == 0):
            best, bd = c, d
    return best


def s_enc(amax: Fraction):
    if amax == 0:
        return Fraction(1)
    s = rn32(Fraction(2688) / amax)
    return FLT_MAX if s is INF else s


def block_sf(ba, s):
    u = rn32(rn32(ba / 6) * s)
    return nearest_even(u, E4M3, 0x7E)


def block_enc(sf, s):
    if sf == 0:
        return Fraction(0)
    e = rn32(s / E4M3[sf])
    return FLT_MAX if e is INF else e


def code(x: Fraction, neg: bool, enc: Fraction) -> int:
    y = rn32(x * enc)
    return (0x8 if neg else 0) | nearest_even(abs(y), E2M1, 7)


def to_fracs(t: torch.Tensor):
    f = t.float().numpy()
    return [[Fraction(float(v)) for v in row] for row in f], np.signbit(f)


def cast_blocks(vals, negs, s):
    """One 16-element block list -> (sf, 8 bytes)."""
    ba = max(abs(v) for v in vals)
    sf = block_sf(ba, s)
    enc = block_enc(sf, s)
    cs = [code(v, n, enc) for v, n in zip(vals, negs)]
    return sf, [cs[2 * j] | (cs[2 * j + 1] << 4) for j in range(8)]


def exact_quantize(t: torch.Tensor):
    X, S = to_fracs(t)
    M, K = len(X), len(X[0])
    amax_row = [max(abs(v) for v in row) for row in X]
    amax_col = [max(abs(X[r][c]) for r in range(M)) for c in range(K)]
    q_row = np.zeros((M, K // 2), np.uint8)
    sf_row = np.zeros((M, K // 16), np.uint8)
    for r in range(M):
        s = s_enc(amax_row[r])
        for b in range(K // 16):
            sf, by = cast_blocks(X[r][16 * b:16 * b + 16], S[r][16 * b:16 * b + 16], s)
            sf_row[r, b] = sf
            q_row[r, 8 * b:8 * b + 8] = by
    q_col = np.zeros((K, M // 2), np.uint8)
    sf_col = np.zeros((K, M // 16), np.uint8)
    for c in range(K):
        s = s_enc(amax_col[c])
        for b in range(M // 16):
            vals = [X[16 * b + i][c] for i in range(16)]
            negs = [S[16 * b + i][c] for i in range(16)]
            sf, by = cast_blocks(vals, negs, s)
            sf_col[c, b] = sf
            q_col[c, 8 * b:8 * b + 8] = by
    return dict(q_row=q_row, sf_row=sf_row, q_col=q_col, sf_col=sf_col,
                amax_row=np.array([float(a) for a in amax_row], np.float32),
                amax_col=np.array([float(a) for a in amax_col], np.float32))


def exact_weight_2d(t: torch.Tensor):
    X, S = to_fracs(t)
    N, K = len(X), len(X[0])
    amax = [max(abs(v) for v in row) for row in X]
    q = np.zeros((N, K // 2), np.uint8)
    sfo = np.zeros((N, K // 16), np.uint8)
    for band in range(N // 16):
        for b in range(K // 16):
            rows = range(16 * band, 16 * band + 16)
            us = [rn32(rn32(max(abs(v) for v in X[r][16 * b:16 * b + 16]) / 6) * s_enc(amax[r])) for r in rows]
            sf = nearest_even(max(us), E4M3, 0x7E)
            for r in rows:
                enc = block_enc(sf, s_enc(amax[r]))
                cs = [code(v, n, enc) for v, n in zip(X[r][16 * b:16 * b + 16], S[r][16 * b:16 * b + 16])]
                q[r, 8 * b:8 * b + 8] = [cs[2 * j] | (cs[2 * j + 1] << 4) for j in range(8)]
                sfo[r, b] = sf
    return dict(q_row=q, sf_row=sfo, amax_row=np.array([float(a) for a in amax], np.float32))


@pytest.mark.parametrize("kind,M,K,seed", [("normal", 32, 48, 0), ("wide", 32, 32, 1), ("tiny", 16, 32, 2),
                                           ("signed_zero", 16, 16, 3)])
def test_exact_rational_matches_oracle(orc, kind, M, K, seed):
    x = inputs.random_shape(seed, M, K, kind)
    want = exact_quantize(x)
    got = orc.quantize(x)
    for k, v in want.items():
        assert np.array_equal(got[k], v), k


def test_exact_rational_matches_oracle_tiny_workload_slice(orc):
    x = inputs.tiny(0)[:32, :64].contiguous()  # contains outlier row 7 and zero row 3
    want = exact_quantize(x)
    got = orc.quantize(x)
    for k, v in want.items():
        assert np.array_equal(got[k], v), k


def test_exact_rational_weight_2d(orc):
    x = inputs.random_shape(4, 32, 32, "wide")
    want = exact_weight_2d(x)
    got = orc.quantize_weight_2d(x)
    for k, v in want.items():
        assert np.array_equal(got[k], v), k
