"""Pins of the oracle's columnwise options (TransformerEngine PR #3045, Changes: opt-in
RHT / SR on the per-token path; review: the row direction never uses RHT). The pages
fix neither the transform nor the random numbers; the readings are in the oracle's
source. What pins each part, independently of the oracle's own code:

* Philox4x32-10: the published known-answer vectors (tests/golden).
* RHT: on small-integer blocks every butterfly sum is exact, so the transform must equal
  (1/4) H16 S v with H16 built here by Kronecker products (H2 (x) H2 (x) H2 (x) H2), and
  applying it twice (no signs) returns the input; Parseval; the sign mask equals
  negating the masked inputs first; on general data it stays within the rounding bound
  of the exact transform.
* SR: the rounding threshold at its exact boundary (r = T - 1 rounds up, r = T down),
  grid values never move, saturation at 6, the sign, and the exact expectation over all
  2^32 random words equals y up to one step of 2^-32 of the E2M1 gap.
* The columnwise cast with RHT equals the plain columnwise cast of the matrix
  transformed here (exactly representable cases); with neither option it equals the
  plain columnwise cast.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from precision_quantization_row_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "philox4x32_10_kat.json")
E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


@pytest.fixture(scope="module", autouse=True)
def _build():
    oracle.build()


def sylvester16() -> np.ndarray:
    h2 = np.array([[1, 1], [1, -1]], np.int64)
    h = h2
    for _ in range(3):
        h = np.kron(h, h2)
    return h


def test_philox_known_answers():
    with open(GOLDEN) as f:
        kat = json.load(f)["vectors"]
    for v in kat:
        ctr = [int(c, 16) for c in v["ctr"]]
        key = [int(k, 16) for k in v["key"]]
        want = [int(o, 16) for o in v["out"]]
        assert oracle.philox4x32_10(ctr, key).tolist() == want


def test_sr_word_uses_counter_and_key():
    seed, off = 0x0123456789ABCDEF, 0x0000000500000007
    for m, k in [(0, 0), (5, 3), (1023, 77), (4, 3)]:
        ctr = [m >> 2, k, off & 0xFFFFFFFF, off >> 32]
        key = [seed & 0xFFFFFFFF, seed >> 32]
        assert oracle.sr_word(m, k, seed, off) == int(oracle.philox4x32_10(ctr, key)[m & 3])


def test_rht_exact_on_small_integers():
    rng = np.random.default_rng(1)
    H = sylvester16()
    for trial in range(200):
        v = rng.integers(-8, 9, 16).astype(np.float32)
        mask = int(rng.integers(0, 1 << 16))
        s = np.array([-1 if (mask >> j) & 1 else 1 for j in range(16)], np.int64)
        want = (H @ (s * v.astype(np.int64))).astype(np.float64) / 4.0
        got = oracle.rht16(v, mask)
        assert np.array_equal(got.astype(np.float64), want), (trial, mask)
        # the mask equals negating the masked inputs first
        assert np.array_equal(got, oracle.rht16((s * v).astype(np.float32), 0))
        # Parseval: (1/4 H16) is orthogonal
        assert float(np.sum(got.astype(np.float64) ** 2)) == float(np.sum(v.astype(np.float64) ** 2))


def test_rht_is_an_involution_without_signs():
    rng = np.random.default_rng(2)
    for _ in range(200):
        v = (rng.integers(-64, 65, 16) * 4).astype(np.float32)   # every stage exact
        assert np.array_equal(oracle.rht16(oracle.rht16(v, 0), 0), v)


def test_rht_within_rounding_bound_on_general_data():
    """Four butterfly stages, each sum or difference rounded once: |v' - exact| is at
    most 4 * 2^-24 * (1/4) * sum |v| (first order), times 1 + 2^-20."""
    rng = np.random.default_rng(3)
    H = sylvester16()
    for _ in range(500):
        v = (rng.standard_normal(16) * np.exp(rng.uniform(-20, 20, 16))).astype(np.float32)
        mask = int(rng.integers(0, 1 << 16))
        s = np.array([-1 if (mask >> j) & 1 else 1 for j in range(16)])
        exact = [sum(Fraction(int(H[i, j] * s[j])) * Fraction(float(v[j])) for j in range(16)) / 4 for i in range(16)]
        got = oracle.rht16(v, mask)
        scale = sum(abs(Fraction(float(t))) for t in v) / 4
        bound = Fraction(4, 1 << 24) * scale * (1 + Fraction(1, 1 << 20))
        for i in range(16):
            assert abs(Fraction(float(got[i])) - exact[i]) <= bound


def _sr_threshold(a: float) -> tuple:
    """(lower code, upper code, T): rounds up iff r < T, T = ceil(f * 2^32), f exact."""
    a = Fraction(a)
    c = max(i for i in range(8) if Fraction(E2M1[i]) <= a)
    lo, hi = Fraction(E2M1[c]), Fraction(E2M1[c + 1])
    f = (a - lo) / (hi - lo)
    t = f * (1 << 32)
    T = -((-t.numerator) // t.denominator)
    return c, c + 1, T


def test_sr_threshold_boundaries():
    rng = np.random.default_rng(4)
    ys = list(rng.uniform(0, 6, 300).astype(np.float32)) + [np.float32(v) for v in (0.25, 0.75, 1.25, 2.5, 5.0,
                                                                                    1e-30, 5.999999)]
    for y in ys:
        lo, hi, T = _sr_threshold(float(y))
        if T > 0:
            assert oracle.e2m1_sr(float(y), T - 1) == hi, y
            assert oracle.e2m1_sr(float(y), 0) == hi, y
        if T < (1 << 32):
            assert oracle.e2m1_sr(float(y), T) == lo, y
            assert oracle.e2m1_sr(float(y), 0xFFFFFFFF) == lo, y


def test_sr_grid_saturation_and_sign():
    for c, v in enumerate(E2M1):
        for r in (0, 1, 0x7FFFFFFF, 0xFFFFFFFF):
            assert oracle.e2m1_sr(v, r) == c
            assert oracle.e2m1_sr(-v, r) == (0x8 | c)
    for y in (6.0, 6.5, 100.0, 3.0e38):
        for r in (0, 0xFFFFFFFF):
            assert oracle.e2m1_sr(y, r) == 7
            assert oracle.e2m1_sr(-y, r) == 0xF
    # a negative value that rounds down to zero keeps its sign
    assert oracle.e2m1_sr(-0.1, 0xFFFFFFFF) == 0x8


def test_sr_expectation_is_exact():
    """Over all 2^32 words the mean of SR(y) is lo + gap * T / 2^32, within gap * 2^-32 of y."""
    rng = np.random.default_rng(5)
    for y in rng.uniform(0, 6, 200).astype(np.float32):
        lo, hi, T = _sr_threshold(float(y))
        gap = Fraction(E2M1[hi]) - Fraction(E2M1[lo])
        mean = Fraction(E2M1[lo]) + gap * Fraction(T, 1 << 32)
        assert abs(mean - Fraction(float(y))) <= gap / (1 << 32)


def test_sr_statistics_with_philox_words():
    """SR with the Philox stream is unbiased in practice: 20000 draws per value."""
    for y in (0.2, 0.7, 1.3, 2.25, 4.9):
        vals = [E2M1[oracle.e2m1_sr(y, oracle.sr_word(m, 7, 42, 0)) & 7] for m in range(20000)]
        lo = max(v for v in E2M1 if v <= y)
        hi = min(v for v in E2M1 if v > y)
        p = (y - lo) / (hi - lo)
        sd = (hi - lo) * (p * (1 - p) / len(vals)) ** 0.5
        assert abs(np.mean(vals) - y) < 5 * sd + 1e-9, y


def test_colwise_opts_without_options_is_the_plain_cast():
    x = inputs.random_shape(41, 96, 48, "wide")
    want = oracle.quantize(x, flags=oracle.COLWISE)
    got = oracle.quantize_colwise_opts(x)
    for k in ("q_col", "sf_col", "amax_col"):
        assert np.array_equal(np.asarray(got[k]).view(np.uint8), np.asarray(want[k]).view(np.uint8)), k


@pytest.mark.parametrize("offsets", [None, [0, 32, 32, 96]], ids=["one_group", "groups"])
def test_colwise_rht_equals_plain_cast_of_transformed_matrix(offsets):
    """Small-integer entries: each transformed value is a multiple of 1/4 below 16, exact
    in bf16, so the RHT cast must equal the plain columnwise cast of (1/4) H16 S applied
    here to every 16-row block of every column."""
    rng = np.random.default_rng(6)
    M, K = 96, 48
    xi = rng.integers(-3, 4, (M, K)).astype(np.float32)
    mask = 0b1011_0110_0101_1100
    H = sylvester16()
    s = np.array([-1 if (mask >> j) & 1 else 1 for j in range(16)])
    xt = np.empty_like(xi)
    for b in range(M // 16):
        blk = xi[16 * b:16 * b + 16].astype(np.int64)
        xt[16 * b:16 * b + 16] = (H @ (s[:, None] * blk)).astype(np.float32) / 4
    x = torch.from_numpy(xi).to(torch.bfloat16)
    xt_b = torch.from_numpy(xt).to(torch.bfloat16)
    assert torch.equal(xt_b.float(), torch.from_numpy(xt))   # exact in bf16
    got = oracle.quantize_colwise_opts(x, offsets=offsets, rht=True, rht_signs=mask)
    if offsets is None:
        want = oracle.quantize(xt_b, flags=oracle.COLWISE)
    else:
        want = oracle.quantize_grouped(xt_b, offsets, flags=oracle.COLWISE)
    for k in ("q_col", "sf_col", "amax_col"):
        assert np.array_equal(np.asarray(got[k]).view(np.uint8), np.asarray(want[k]).view(np.uint8)), k


def test_colwise_sr_codes_are_neighbours_of_the_rn_codes():
    """SR picks one of the two E2M1 neighbours of each scaled value; RN picks the nearer,
    so the two codes are equal or adjacent with the same sign. Scales and amax agree."""
    x = inputs.random_shape(43, 64, 32, "normal")
    rn = oracle.quantize_colwise_opts(x)
    sr = oracle.quantize_colwise_opts(x, sr=True, seed=7, offset=1)
    assert np.array_equal(rn["sf_col"], sr["sf_col"])
    assert np.array_equal(rn["amax_col"].view(np.uint32), sr["amax_col"].view(np.uint32))
    for q in (rn["q_col"], sr["q_col"]):
        assert q.shape == (32, 32)
    a = np.stack([rn["q_col"] & 0xF, rn["q_col"] >> 4], -1)
    b = np.stack([sr["q_col"] & 0xF, sr["q_col"] >> 4], -1)
    nz = (a & 7) != 0
    assert np.all(((a & 8) == (b & 8)) | ~nz)
    assert np.all(np.abs((a & 7).astype(int) - (b & 7).astype(int)) <= 1)
    assert not np.array_equal(a, b)   # some values did round the other way
    again = oracle.quantize_colwise_opts(x, sr=True, seed=7, offset=1)
    assert np.array_equal(sr["q_col"], again["q_col"])
    other = oracle.quantize_colwise_opts(x, sr=True, seed=7, offset=2)
    assert not np.array_equal(sr["q_col"], other["q_col"])
