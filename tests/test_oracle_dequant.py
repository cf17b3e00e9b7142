"""Pins of the oracle's dequantization and columnwise requantization, each against
something other than the oracle's own formula: torch's bf16 conversion, closed forms
where the decode scale is a power of two, the NVFP4 error bound of the round trip,
and a lossless construction where requantizing must reproduce the direct cast."""
import numpy as np
import pytest
import torch

E4M3_FINITE = [c for c in range(0x7F)]   # non-negative finite E4M3 codes (0x7F is NaN)


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_bf16_rounding_matches_torch(orc):
    rng = np.random.default_rng(50)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 20000),
        # exact ties: a bf16 value plus half its last place, both parities
        (np.arange(0x3F80, 0x3F80 + 256, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        -(np.arange(0x0080, 0x0080 + 256, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([0.0, -0.0, 1e-45, -1e-45, 3.3e38, -3.3e38], np.float32),
        # the top of the range: below, at and above halfway from the largest finite bf16
        # (0x7F7F) to 2^128, where rounding to nearest overflows to infinity
        np.array([0x7F7F7FFF, 0x7F7F8000, 0x7F7F8001, 0x7F7FFFFF, 0x7F7EFFFF, 0xFF7F8000, 0xFF7F7FFF,
                  0x7F800000, 0xFF800000], np.uint32).view(np.float32),
    ])
    assert np.array_equal(orc.f32_to_bf16(v), _bf16_bits(torch.from_numpy(v)))


def _random_nvfp4(rng, M, K):
    q = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    sf = rng.choice(E4M3_FINITE, (M, K // 16)).astype(np.uint8)
    return q, sf


def _expected_products(orc, q, sf):
    """val(code) * float(sf) per element with the pinned decode tables, element 2j
    taken from the low nibble of byte j (float64: exact)."""
    M, half = q.shape
    codes = np.empty((M, 2 * half), np.uint8)
    codes[:, 0::2] = q & 0xF
    codes[:, 1::2] = q >> 4
    e2 = np.array([orc.e2m1_decode(c) for c in range(16)], np.float64)
    e4 = np.array([orc.e4m3_decode(c) for c in range(256)], np.float64)
    return e2[codes] * e4[sf].repeat(16, axis=1)


@pytest.mark.parametrize("k", [0, -20, 7, 100])
def test_dequant_power_of_two_decode_scale(orc, k):
    """amax = 2688 * 2^k: the decode scale amax/2688 is exactly 2^k, so every output is
    val(q) * float(sf) * 2^k, which bf16 holds exactly (at most 6 significant bits)."""
    rng = np.random.default_rng(51 + k)
    M, K = 32, 64
    q, sf = _random_nvfp4(rng, M, K)
    amax = np.full(M, np.float32(2688.0 * 2.0 ** k))
    want = (_expected_products(orc, q, sf) * 2.0 ** k).astype(np.float32)
    assert np.array_equal(orc.dequantize(q, sf, amax), _bf16_bits(torch.from_numpy(want)))


def test_dequant_zero_amax_gives_signed_zeros(orc):
    rng = np.random.default_rng(52)
    q, sf = _random_nvfp4(rng, 16, 32)
    got = orc.dequantize(q, sf, np.zeros(16, np.float32))
    codes = np.empty((16, 32), np.uint8)
    codes[:, 0::2] = q & 0xF
    codes[:, 1::2] = q >> 4
    neg = (codes & 0x8) != 0
    assert np.array_equal(got, np.where(neg, 0x8000, 0x0000).astype(np.uint16))


@pytest.mark.parametrize("kind", ["normal", "wide"])
def test_round_trip_within_nvfp4_bound(orc, kind):
    """dequantize(quantize(x)) is within half an E2M1 step of x in the block's unit
    (float(sf) * amax/2688), plus the bf16 rounding of the result. (Rows whose amax
    is below ~7.9e-36 are outside this bound by the cast's own reading: their s_enc is
    clamped to FLT_MAX, so amax/2688 no longer inverts it.)"""
    from precision_quantization_row_b200 import inputs
    x = inputs.random_shape(53, 64, 256, kind)
    out = orc.quantize(x)
    got = torch.from_numpy(orc.dequantize(out["q_row"], out["sf_row"], out["amax_row"]).view(np.int16))
    xd = got.view(torch.bfloat16).double().numpy()
    xf = x.double().numpy()
    amax = out["amax_row"].astype(np.float64)[:, None]
    unit = np.array([orc.e4m3_decode(c) for c in range(256)])[out["sf_row"]].repeat(16, axis=1) * amax / 2688.0
    y = np.divide(np.abs(xf), unit, out=np.zeros_like(xf), where=unit > 0)
    half_step = np.where(y < 2.0, 0.25, np.where(y < 4.0, 0.5, 1.0))
    bound = half_step * unit * (1 + 2.0 ** -10) + np.abs(xd) * 2.0 ** -8 + 1e-300
    assert np.all(np.abs(xd - xf) <= bound)


def _lossless_matrix(rng, M, K, groups_ok=True):
    """A bf16 matrix whose rowwise cast is lossless: row r has amax 6 * 448 * 2^k_r
    (a code 6 in a block of scale 448), every block holds a +-6, and every value is
    val * sf * 2^k_r with val an E2M1 value and sf an E4M3 value."""
    e2 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    e4 = np.array([(1 + (c & 7) / 8) * 2.0 ** ((c >> 3) - 7) if c >> 3 else (c & 7) * 2.0 ** -9
                   for c in range(0x7F)])
    x = np.empty((M, K))
    for r in range(M):
        k = int(rng.integers(-8, 8))
        sf = e4[rng.integers(40, 0x7F, K // 16)]
        sf[rng.integers(0, K // 16)] = 448.0
        vals = e2[rng.integers(0, 8, K)] * rng.choice([-1.0, 1.0], K)
        vals[16 * np.arange(K // 16) + rng.integers(0, 16, K // 16)] = 6.0 * rng.choice([-1.0, 1.0], K // 16)
        x[r] = vals * sf.repeat(16) * 2.0 ** k
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)


def test_requant_of_lossless_rows_is_the_direct_columnwise_cast(orc):
    rng = np.random.default_rng(54)
    x = _lossless_matrix(rng, 64, 96)
    rows = orc.quantize(x, flags=1)
    xd = orc.dequantize(rows["q_row"], rows["sf_row"], rows["amax_row"])
    assert np.array_equal(xd, x.view(torch.int16).numpy().view(np.uint16))   # lossless indeed
    got = orc.requantize_colwise(rows["q_row"], rows["sf_row"], rows["amax_row"], absmax=np.zeros(1, np.float32),
                                 decay=0.5)
    want = orc.quantize(x, flags=2, absmax=0.0, decay=0.5)
    for key in ("q_col", "sf_col", "amax_col"):
        assert np.array_equal(got[key], want[key]), key
    assert np.float32(got["absmax"][0]) == np.float32(want["absmax"])


def test_grouped_requant_of_lossless_rows(orc):
    rng = np.random.default_rng(55)
    x = _lossless_matrix(rng, 96, 48)
    offsets = [0, 32, 32, 80, 96]
    rows = orc.quantize(x, flags=1)
    got = orc.requantize_colwise(rows["q_row"], rows["sf_row"], rows["amax_row"], offsets=offsets)
    want = orc.quantize_grouped(x, offsets, flags=2)
    for key in ("q_col", "sf_col", "amax_col"):
        assert np.array_equal(got[key], want[key]), key
