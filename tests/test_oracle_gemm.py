"""Pins of the oracle's per-token NVFP4 GEMM, each against something other than its
own formula: exact rational arithmetic on tiny operands (E2M1 and e4m3fn values
written out here from the formats' bit fields), integer matrix products where every
value is a small integer, products that power-of-two block scales and amaxes shift
exactly, the symmetry D(A, B) = D(B, A)^T, and the pinned cast and dequantization
(the GEMM of two cast matrices is the product of their dequantizations up to the
bf16 rounding of the latter)."""
from fractions import Fraction

import numpy as np
import pytest

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # magnitude of each 3-bit E2M1 index
F32 = np.float32


def _pack(codes: np.ndarray) -> np.ndarray:
    """[R, K] 4-bit codes -> [R, K/2] bytes, element 2j in the low nibble."""
    codes = np.asarray(codes, np.uint8)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def _e2m1_value(c: int) -> Fraction:
    v = Fraction(E2M1[c & 7])
    return -v if c & 8 else v


def _e4m3_value(c: int) -> Fraction:
    """e4m3fn value of a non-negative code from its fields (bias 7; exponent 0 is subnormal)."""
    e, m = (c >> 3) & 0xF, c & 7
    return Fraction(m, 512) if e == 0 else Fraction(8 + m, 8) * Fraction(2) ** (e - 7)


def _decode_scale(amax) -> Fraction:
    return Fraction(float(F32(amax) / F32(2688.0)))   # one binary32 division, nearest-even


# the last case draws only subnormal block scales (e4m3fn codes 0..7)
@pytest.mark.parametrize("M,N,K,top", [(1, 1, 16, 0x7F), (3, 4, 32, 0x7F), (5, 2, 64, 0x7F), (2, 3, 48, 8)])
def test_gemm_equals_exact_rational_sum(orc, M, N, K, top):
    rng = np.random.default_rng(90 + K)
    ca, cb = rng.integers(0, 16, (M, K)), rng.integers(0, 16, (N, K))
    sa, sb = rng.integers(0, top, (M, K // 16)), rng.integers(0, top, (N, K // 16))
    aa = np.abs(rng.standard_normal(M) * 10.0 ** rng.integers(-3, 4, M)).astype(F32)
    ab = np.abs(rng.standard_normal(N) * 10.0 ** rng.integers(-3, 4, N)).astype(F32)
    d, mag = orc.gemm_per_token(_pack(ca), sa.astype(np.uint8), aa, _pack(cb), sb.astype(np.uint8), ab)
    for m in range(M):
        for n in range(N):
            terms = [_e2m1_value(int(ca[m, k])) * _e4m3_value(int(sa[m, k // 16])) *
                     _e2m1_value(int(cb[n, k])) * _e4m3_value(int(sb[n, k // 16])) for k in range(K)]
            scale = _decode_scale(aa[m]) * _decode_scale(ab[n])
            exact, exact_mag = sum(terms) * scale, sum(abs(t) for t in terms) * scale
            # the sum is exact; the result takes two double roundings
            assert abs(Fraction(d[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 50), (m, n)
            assert abs(Fraction(mag[m, n]) - exact_mag) <= exact_mag * Fraction(1, 2 ** 50), (m, n)


def _integer_operand(rng, R, K):
    """Codes whose values are the integers 0, +-1, +-2, +-3, +-4, +-6, and those values."""
    idx = np.array([0, 2, 4, 5, 6, 7])[rng.integers(0, 6, (R, K))]
    neg = rng.integers(0, 2, (R, K)).astype(np.uint8)
    vals = np.array(E2M1)[idx] * np.where(neg == 1, -1.0, 1.0)
    return (idx | (neg << 3)).astype(np.uint8), vals.astype(np.int64)


def test_gemm_of_integer_values_is_the_integer_product(orc):
    """Scales 1.0 (e4m3fn 0x38) and amax 2688 (decode scale 1): D = Va Vb^T exactly."""
    rng = np.random.default_rng(91)
    M, N, K = 33, 17, 256
    ca, va = _integer_operand(rng, M, K)
    cb, vb = _integer_operand(rng, N, K)
    d, _ = orc.gemm_per_token(_pack(ca), np.full((M, K // 16), 0x38, np.uint8), np.full(M, 2688.0, F32),
                              _pack(cb), np.full((N, K // 16), 0x38, np.uint8), np.full(N, 2688.0, F32))
    assert np.array_equal(d, (va @ vb.T).astype(np.float64))


def test_power_of_two_scales_shift_block_products_exactly(orc):
    """Block scales 2^k (e4m3fn exponent field 7 + k) and amaxes 2688 * 2^j: each
    block's integer product is shifted by its two scales, each row and column by j."""
    rng = np.random.default_rng(92)
    M, N, K = 8, 6, 128
    nb = K // 16
    ca, va = _integer_operand(rng, M, K)
    cb, vb = _integer_operand(rng, N, K)
    ka, kb = rng.integers(-6, 7, (M, nb)), rng.integers(-6, 7, (N, nb))
    ja, jb = rng.integers(-5, 6, M), rng.integers(-5, 6, N)
    d, _ = orc.gemm_per_token(_pack(ca), (0x38 + 8 * ka).astype(np.uint8), (2688.0 * 2.0 ** ja).astype(F32),
                              _pack(cb), (0x38 + 8 * kb).astype(np.uint8), (2688.0 * 2.0 ** jb).astype(F32))
    block = np.einsum("mbi,nbi->mnb", va.reshape(M, nb, 16), vb.reshape(N, nb, 16)).astype(np.float64)
    shift = 2.0 ** (ka[:, None, :] + kb[None, :, :])
    want = (block * shift).sum(axis=2) * 2.0 ** (ja[:, None] + jb[None, :])
    assert np.array_equal(d, want)


def test_gemm_is_symmetric_in_its_operands(orc):
    rng = np.random.default_rng(93)
    M, N, K = 7, 9, 96
    qa, qb = rng.integers(0, 256, (M, K // 2), dtype=np.uint8), rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = rng.integers(0, 0x7F, (M, K // 16)).astype(np.uint8)
    sb = rng.integers(0, 0x7F, (N, K // 16)).astype(np.uint8)
    aa, ab = rng.uniform(0.1, 50, M).astype(F32), rng.uniform(0.1, 50, N).astype(F32)
    d1, m1 = orc.gemm_per_token(qa, sa, aa, qb, sb, ab)
    d2, m2 = orc.gemm_per_token(qb, sb, ab, qa, sa, aa)
    assert np.array_equal(d1, d2.T) and np.array_equal(m1, m2.T)


def test_gemm_of_cast_matrices_is_the_product_of_their_dequantizations(orc):
    """D(cast(X), cast(W)) against dequantize(X) dequantize(W)^T in float64: each
    dequantized element is the GEMM's exact val*sf*S_dec rounded to binary32 and then
    to bf16 (relative error below 2^-9 + 2^-24), so the two differ by less than
    2 (2^-9 + 2^-24) + its square times the magnitudes' sum. A transposed operand, a
    wrong block index or a missing decode scale gives errors of that sum's order."""
    import torch

    from precision_quantization_row_b200 import inputs
    x = inputs.random_shape(94, 48, 256, "normal")
    w = inputs.random_shape(95, 32, 256, "wide")
    rx, rw = orc.quantize(x, flags=orc.ROWWISE), orc.quantize(w, flags=orc.ROWWISE)
    d, mag = orc.gemm_per_token(rx["q_row"], rx["sf_row"], rx["amax_row"], rw["q_row"], rw["sf_row"], rw["amax_row"])

    def deq(r):
        bits = orc.dequantize(r["q_row"], r["sf_row"], r["amax_row"])
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()

    ref = deq(rx) @ deq(rw).T
    u = 2.0 ** -9 + 2.0 ** -24
    assert np.all(np.abs(d - ref) <= (2 * u + u * u) * mag * (1 + 2.0 ** -40))
    # and the cast matrices' product is close to X W^T itself (NVFP4: a few percent)
    xw = x.double().numpy() @ w.double().numpy().T
    assert np.abs(d - xw).max() <= 0.1 * np.abs(x.double().numpy()).sum(1).max() * np.abs(w.double().numpy()).max()


def test_zero_amax_rows_and_columns(orc):
    rng = np.random.default_rng(96)
    M, N, K = 4, 3, 32
    qa, qb = rng.integers(0, 256, (M, K // 2), dtype=np.uint8), rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = rng.integers(1, 0x7F, (M, K // 16)).astype(np.uint8)
    sb = rng.integers(1, 0x7F, (N, K // 16)).astype(np.uint8)
    aa, ab = np.array([0, 1, 2, 0], F32), np.array([3, 0, 5], F32)
    d, mag = orc.gemm_per_token(qa, sa, aa, qb, sb, ab)
    assert np.all(d[[0, 3], :] == 0) and np.all(d[:, 1] == 0)
    assert np.all(mag[[0, 3], :] == 0) and np.all(mag[:, 1] == 0)


def test_rejections(orc):
    q = np.zeros((2, 8), np.uint8)
    s = np.full((2, 1), 0x38, np.uint8)
    a = np.ones(2, F32)
    with pytest.raises(ValueError):
        orc.gemm_per_token(q, np.full((2, 1), 0x7F, np.uint8), a, q, s, a)   # NaN scale
    with pytest.raises(ValueError):
        orc.gemm_per_token(q, s, a, q, np.full((2, 1), 0x80, np.uint8), a)   # negative scale code
    with pytest.raises(ValueError):
        orc.gemm_per_token(q, s, a, np.zeros((2, 16), np.uint8), np.full((2, 2), 0x38, np.uint8), a)   # K differs
    with pytest.raises(ValueError):
        orc.gemm_per_token(np.zeros((2, 4), np.uint8), np.zeros((2, 0), np.uint8), a,
                           np.zeros((2, 4), np.uint8), np.zeros((2, 0), np.uint8), a)   # K = 8


def test_sum_is_exact_where_a_double_accumulation_rounds(orc):
    """K = 8192: 511 blocks of codes 6 at scale 448 push the running sum to about 2^55.8
    units of 2^-20; a last block of +-0.5 and +-1.5 at subnormal scales adds terms of a
    few units, which a double accumulation rounds away (checked here on the same data).
    The oracle must equal the exact integer sum (Python integers), rounded once."""
    rng = np.random.default_rng(97)
    M, N, K = 2, 3, 8192
    nb = K // 16

    def operand(R):
        codes = np.full((R, K), 7)                                    # 6.0
        codes[:, K - 16:] = rng.choice([1, 3, 9, 11], (R, 16))       # +-0.5, +-1.5
        sf = np.full((R, nb), 0x7E)                                   # 448
        sf[:, nb - 1] = rng.integers(1, 8, R)                         # subnormal: m * 2^-9
        return codes, sf

    (ca, sa), (cb, sb) = operand(M), operand(N)
    aa, ab = np.full(M, 2688.0, F32), np.full(N, 2688.0, F32)   # decode scale 1
    d, _ = orc.gemm_per_token(_pack(ca), sa.astype(np.uint8), aa, _pack(cb), sb.astype(np.uint8), ab)
    twice = [0, 1, 2, 3, 4, 6, 8, 12]
    sf512 = [int(_e4m3_value(c) * 512) for c in range(0x7F)]
    for m in range(M):
        for n in range(N):
            units, as_double = 0, 0.0   # in 2^-20
            for k in range(K):
                va, vb = twice[ca[m, k] & 7], twice[cb[n, k] & 7]
                t = (-va if ca[m, k] & 8 else va) * (-vb if cb[n, k] & 8 else vb)
                t *= sf512[sa[m, k // 16]] * sf512[sb[n, k // 16]]
                units += t
                as_double += t
            assert abs(units) > 2 ** 53 and as_double != units   # the regime where doubles round
            assert d[m, n] == float(Fraction(units, 2 ** 20)), (m, n)
