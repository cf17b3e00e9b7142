"""Pins of the oracle's E2M1 and E4M3 conversions against things other than itself.

The formats are the OCP FP4 E2M1 and FP8 E4M3 (e4m3fn) encodings that NVFP4 uses
(TransformerEngine PR #3045 "Add NVFP4 per-token quantization recipe", Changes:
E2M1 codes with E4M3 block scales). The checks here:
  * every code decodes to the value its bit fields define, and re-encodes to itself;
  * every midpoint between neighbours goes to the even code, and the floats just
    above/below it go to the upper/lower neighbour (round-to-nearest-even);
  * saturation above the largest finite value (E2M1: 6, E4M3: 448);
  * agreement with two independent libraries (ml_dtypes, and torch's float8_e4m3fn)
    over every bf16 value, dense float32 neighbourhoods of every midpoint and
    random float32 samples.
"""
import math

import ml_dtypes
import numpy as np
import pytest
import torch


def e2m1_value_from_bits(code: int) -> float:
    """OCP E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; exponent 0 is subnormal."""
    s = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    mag = m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return s * mag


def e4m3_value_from_bits(code: int) -> float:
    """OCP E4M3 (fn): 1 sign, 4 exponent (bias 7), 3 mantissa bits; S.1111.111 is NaN."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    mag = math.ldexp(m / 8.0, -6) if e == 0 else math.ldexp(1.0 + m / 8.0, e - 7)
    return s * mag


E4M3_FINITE = [c for c in range(256) if (c & 0x7F) != 0x7F]


def test_e2m1_decode_matches_bit_fields(orc):
    for c in range(16):
        assert orc.e2m1_decode(c) == e2m1_value_from_bits(c)
        assert math.copysign(1.0, orc.e2m1_decode(c)) == math.copysign(1.0, e2m1_value_from_bits(c)) or c in (0, 8)


def test_e2m1_roundtrip_every_code(orc):
    for c in range(16):
        v = e2m1_value_from_bits(c)
        if c == 8:
            v = -0.0
        assert orc.e2m1(v) == c, (c, v)


def test_e4m3_decode_matches_bit_fields_and_libraries(orc):
    codes = np.array(E4M3_FINITE, np.uint8)
    torch_vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    mld_vals = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    for i, c in enumerate(E4M3_FINITE):
        want = e4m3_value_from_bits(c)
        assert orc.e4m3_decode(c) == want
        assert torch_vals[i] == want and mld_vals[i] == want


def test_e4m3_roundtrip_every_finite_code(orc):
    for c in E4M3_FINITE:
        v = e4m3_value_from_bits(c)
        if c == 0x80:
            v = -0.0
        assert orc.e4m3(v) == c, hex(c)


def _midpoint_checks(values_codes, enc, max_code_lsb_even=True):
    """values_codes: sorted (value, code) pairs of one sign. Checks tie -> even code and
    that the adjacent float32s fall to the nearer neighbour."""
    for (v0, c0), (v1, c1) in zip(values_codes, values_codes[1:]):
        mid = (v0 + v1) / 2.0
        assert np.float32(mid) == mid  # every midpoint is exact in binary32
        even = c0 if (c0 & 1) == 0 else c1
        assert enc(mid) == even, (v0, v1)
        up = float(np.nextafter(np.float32(mid), np.float32(np.inf)))
        dn = float(np.nextafter(np.float32(mid), np.float32(-np.inf)))
        assert enc(up) == c1 and enc(dn) == c0, (v0, v1)


def test_e2m1_ties_to_even_and_neighbours(orc):
    pos = [(e2m1_value_from_bits(c), c) for c in range(8)]
    _midpoint_checks(pos, orc.e2m1)
    neg = [(-v, c | 0x8) for v, c in pos]
    for (v0, c0), (v1, c1) in zip(neg, neg[1:]):
        mid = (v0 + v1) / 2.0
        even = c0 if (c0 & 1) == 0 else c1
        assert orc.e2m1(mid) == even


def test_e4m3_ties_to_even_and_neighbours(orc):
    pos = sorted((e4m3_value_from_bits(c), c) for c in range(0x7F))
    _midpoint_checks(pos, orc.e4m3)


def test_saturation(orc):
    for y in [6.0000005, 6.5, 7.0, 1e30, float("inf")]:
        assert orc.e2m1(y) == 0x7 and orc.e2m1(-y) == 0xF
    assert orc.e2m1(6.0) == 0x7 and orc.e2m1(5.0) == 0x6 and orc.e2m1(5.0000005) == 0x7
    for v in [448.00003, 460.0, 464.0, 1000.0, 3.4e38, float("inf")]:
        assert orc.e4m3(v) == 0x7E
    # 432 is the midpoint of 416 (0x7D, odd) and 448 (0x7E, even)
    assert orc.e4m3(448.0) == 0x7E and orc.e4m3(432.0) == 0x7E and orc.e4m3(431.99997) == 0x7D


def test_signed_zero_and_tiny(orc):
    assert orc.e2m1(0.0) == 0 and orc.e2m1(-0.0) == 8
    assert orc.e2m1(-0.25) == 8 and orc.e2m1(-1e-40) == 8 and orc.e2m1(1e-40) == 0
    assert orc.e4m3(0.0) == 0 and orc.e4m3(2.0 ** -10) == 0  # tie 0|2^-9 -> even code 0
    assert orc.e4m3(float(np.nextafter(np.float32(2.0 ** -10), np.float32(1)))) == 1
    assert orc.e4m3(1e-40) == 0


def _samples():
    rng = np.random.default_rng(1234)
    bf16_all = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    bf16_all = bf16_all[np.isfinite(bf16_all)]
    rand_bits = rng.integers(0, 2 ** 32, 2_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    rand_bits = rand_bits[np.isfinite(rand_bits)]
    logu = (np.exp2(rng.uniform(-12, 10, 2_000_000)) * rng.choice([-1, 1], 2_000_000)).astype(np.float32)
    return np.concatenate([bf16_all, rand_bits, logu])


def _neighbourhoods(values, width=2048):
    """All float32s within `width` ulps of each value (both signs)."""
    out = []
    for v in values:
        b = np.array([v], np.float32).view(np.int32)[0]
        bits = np.arange(b - width, b + width + 1, dtype=np.int64)
        bits = bits[(bits >= 0) & (bits < 0x7F800000)].astype(np.int32)
        f = bits.view(np.float32)
        out.append(f)
        out.append(-f)
    return np.concatenate(out)


def test_e2m1_matches_ml_dtypes(orc):
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0]
    xs = np.concatenate([_samples(), _neighbourhoods(mids, 1 << 14)])
    ours = orc.e2m1_array(xs)
    lib = xs.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    bad = np.nonzero(ours != lib)[0]
    assert bad.size == 0, (xs[bad[:5]], ours[bad[:5]], lib[bad[:5]])


def test_e4m3_matches_libraries_in_range(orc):
    vals = sorted(e4m3_value_from_bits(c) for c in range(0x7F))
    mids = [(a + b) / 2 for a, b in zip(vals, vals[1:])]
    xs = np.concatenate([_samples(), _neighbourhoods(mids, 512)])
    xs = xs[np.abs(xs) <= 448.0]  # the libraries do not saturate; ours does
    ours = orc.e4m3_array(xs)
    mld = xs.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    tch = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero((ours != mld) | (ours != tch))[0]
    assert bad.size == 0, (xs[bad[:5]], ours[bad[:5]], mld[bad[:5]], tch[bad[:5]])


@pytest.mark.parametrize("binade", range(-3, 3))
def test_e2m1_exhaustive_binade(orc, binade):
    """Every positive float32 in [2^b, 2^(b+1)) for the binades where E2M1 decisions happen."""
    lo = np.array([2.0 ** binade], np.float32).view(np.uint32)[0]
    bits = np.arange(lo, lo + (1 << 23), dtype=np.uint32)
    xs = bits.view(np.float32)
    ours = orc.e2m1_array(xs)
    lib = xs.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(ours, lib)
