"""Invariants and closed forms the oracle must satisfy, whatever its internals.

Each property follows from the definition of the per-token cast (TransformerEngine
PR #3045 "Add NVFP4 per-token quantization recipe", Description and Changes) and
would fail for a plausible implementation mistake:
  * columnwise(X) == rowwise(X^T)            -> transposed operand / wrong index
  * codes(-X) == codes(X) ^ 0x88             -> sign handling, sign of zero
  * X * 2^k leaves codes and scales unchanged -> dropped or misplaced scale factor
  * a row with one nonzero a: its code is +-6 -> s_enc / enc formula
  * every code is a nearest E2M1 value of x*enc, and float(sf) is within one E4M3
    rounding of block_amax/6*s_enc            -> the round-trip error bound
  * grouped == ungrouped per token group; weight-2D scale == max of the 1D scales;
    weight-2D is transposition-invariant when all row and column amaxes agree
    (PR #3045, Changes: "transposition-invariant 16x16 cast").
"""
import numpy as np
import pytest
import torch

from precision_quantization_row_b200 import inputs


def _flip_nibbles(a):
    return a ^ np.uint8(0x88)


@pytest.mark.parametrize("seed,M,K", [(0, 32, 48), (1, 64, 64), (2, 48, 128)])
def test_columnwise_is_rowwise_of_transpose(orc, seed, M, K):
    x = inputs.random_shape(seed, M, K, "wide")
    a = orc.quantize(x)
    b = orc.quantize(x.t().contiguous(), flags=orc.ROWWISE)
    assert np.array_equal(a["q_col"], b["q_row"])
    assert np.array_equal(a["sf_col"], b["sf_row"])
    assert np.array_equal(a["amax_col"], b["amax_row"])


@pytest.mark.parametrize("kind", ["normal", "wide", "signed_zero"])
def test_sign_flip(orc, kind):
    x = inputs.random_shape(3, 32, 64, kind)
    a = orc.quantize(x)
    b = orc.quantize(-x)
    for k in ("q_row", "q_col"):
        assert np.array_equal(_flip_nibbles(a[k]), b[k])
    for k in ("sf_row", "sf_col", "amax_row", "amax_col"):
        assert np.array_equal(a[k], b[k])


@pytest.mark.parametrize("k", [-7, -1, 1, 5])
def test_power_of_two_scaling(orc, k):
    x = inputs.random_shape(4, 32, 64, "normal")
    a = orc.quantize(x)
    b = orc.quantize((x.float() * 2.0 ** k).to(torch.bfloat16))
    for key in ("q_row", "q_col", "sf_row", "sf_col"):
        assert np.array_equal(a[key], b[key]), key
    assert np.array_equal(a["amax_row"] * np.float32(2.0 ** k), b["amax_row"])


def test_zero_rows_and_columns(orc):
    x = inputs.random_shape(5, 32, 48, "normal").float()
    x[5] = 0.0
    x[:, 17] = 0.0
    out = orc.quantize(x.to(torch.bfloat16))
    assert out["amax_row"][5] == 0 and not out["q_row"][5].any() and not out["sf_row"][5].any()
    assert out["amax_col"][17] == 0 and not out["q_col"][17].any() and not out["sf_col"][17].any()


def test_single_nonzero_row(orc):
    rng = np.random.default_rng(6)
    vals = (rng.choice([-1.0, 1.0], 64) * np.exp2(rng.uniform(-60, 60, 64))).astype(np.float32)
    x = np.zeros((64, 32), np.float32)
    cols = rng.integers(0, 32, 64)
    x[np.arange(64), cols] = vals
    xb = torch.from_numpy(x).to(torch.bfloat16)
    out = orc.quantize(xb, flags=orc.ROWWISE)
    for r in range(64):
        c = cols[r]
        assert out["sf_row"][r, c // 16] == 0x7E
        other = out["sf_row"][r, 1 - c // 16]
        assert other == 0
        byte = out["q_row"][r, c // 2]
        code = (byte >> 4) if c % 2 else (byte & 0xF)
        assert code == (0xF if vals[r] < 0 else 0x7)
        q = out["q_row"][r].copy()
        q[c // 2] &= np.uint8(0x0F if c % 2 else 0xF0)
        assert not q.any()


def _e2m1_half_spacing(a):
    return np.where(a <= 2.0, 0.25, np.where(a <= 4.0, 0.5, 1.0))


@pytest.mark.parametrize("kind", ["normal", "wide"])
def test_round_trip_bound(orc, kind):
    """Codes are nearest E2M1 values of x*enc, and scales are one E4M3 rounding of
    block_amax/6*s_enc (exact checks in float64 with binary32 rounding slack)."""
    M, K = 64, 96
    x = inputs.random_shape(7, M, K, kind)
    out = orc.quantize(x, flags=orc.ROWWISE)
    xf = x.double().numpy()
    table = np.array([orc.e2m1_decode(c) for c in range(16)])
    codes = np.empty((M, K), np.uint8)
    codes[:, 0::2] = out["q_row"] & 0xF
    codes[:, 1::2] = out["q_row"] >> 4
    q = table[codes]
    amax = np.abs(xf).max(axis=1)
    s = np.where(amax == 0, 1.0, 2688.0 / np.where(amax == 0, 1.0, amax))[:, None]
    d = np.array([orc.e4m3_decode(int(c)) for c in out["sf_row"].ravel()]).reshape(M, K // 16)
    ba = np.abs(xf).reshape(M, K // 16, 16).max(axis=2)
    target = ba / 6.0 * s  # exact real-number scale argument
    rel = np.abs(d - target) / np.where(target == 0, 1, target)
    # one E4M3 rounding (<= 1/16 relative for normals, 2^-10 absolute for subnormals), or saturated at 448
    ok_sf = (rel <= 1 / 16 + 1e-6) | (np.abs(d - target) <= 2.0 ** -10 + 1e-12) | ((d == 448.0) & (target >= 432.0))
    assert ok_sf.all()
    enc = np.where(d == 0, 0.0, s / np.where(d == 0, 1, d)).repeat(16, axis=1)
    y = xf * enc
    a = np.abs(y)
    err = np.abs(y - q)
    slack = 2.0 ** -20 * a + 1e-30
    ok = np.where(a > 6.0, np.abs(q) == 6.0, err <= _e2m1_half_spacing(a) + slack)
    assert ok.all()
    same_sign = (np.sign(q) == np.sign(y)) | (q == 0)
    assert same_sign.all()
    # dequantised value within half an E2M1 step (in the block's scale) of x
    deq = orc.dequantize_rows(out["q_row"], out["sf_row"], out["amax_row"])
    near = np.abs(xf - deq) <= (_e2m1_half_spacing(a) + slack) / np.where(enc == 0, 1, enc) * (1 + 2.0 ** -20)
    saturated = np.abs(deq) <= np.abs(xf) * (1 + 2.0 ** -20)  # clipped towards zero, never beyond x
    assert np.where(a > 6.0, saturated, near).all()


def test_absmax_tiny_stream(orc):
    """Tiny workload, seeds 0..9 at decay 0.9: the buffer equals the decayed running max of max|X|."""
    buf = 0.0
    for s in range(10):
        x = inputs.tiny(s)
        out = orc.quantize(x, absmax=buf, decay=0.9)
        obs = float(x.float().abs().max())
        assert out["amax_row"].max() == obs
        want = max(float(np.float32(buf) * np.float32(0.9)), obs)
        assert out["absmax"] == np.float32(want)
        buf = out["absmax"]


# --------------------------------------------------------------- grouped

@pytest.mark.parametrize("offsets", [[0, 48], [0, 16, 16, 48], [0, 0, 32, 48, 48], [0, 48, 48]])
def test_grouped_equals_ungrouped_per_group(orc, offsets):
    M, K = 48, 64
    x = inputs.random_shape(8, M, K, "wide")
    g = orc.quantize_grouped(x, offsets, absmax=np.full(len(offsets) - 1, 2.0, np.float32), decay=0.5)
    whole = orc.quantize(x, flags=orc.ROWWISE)
    assert np.array_equal(g["q_row"], whole["q_row"]) and np.array_equal(g["sf_row"], whole["sf_row"])
    assert np.array_equal(g["amax_row"], whole["amax_row"])
    for i in range(len(offsets) - 1):
        r0, r1 = offsets[i], offsets[i + 1]
        m = r1 - r0
        if m == 0:
            assert not g["amax_col"][i].any()
            assert g["absmax"][i] == 1.0  # decayed, nothing observed
            continue
        part = orc.quantize(x[r0:r1].contiguous(), flags=orc.COLWISE)
        assert np.array_equal(g["amax_col"][i], part["amax_col"])
        qc = g["q_col"][K * r0 // 2: K * r1 // 2].reshape(K, m // 2)
        sc = g["sf_col"][K * r0 // 16: K * r1 // 16].reshape(K, m // 16)
        assert np.array_equal(qc, part["q_col"]) and np.array_equal(sc, part["sf_col"])
        assert g["absmax"][i] == max(1.0, float(part["amax_col"].max()))


def test_grouped_rejects_bad_offsets(orc):
    x = inputs.random_shape(9, 32, 32)
    for off in ([0, 8, 32], [0, 32, 16, 32], [16, 32], [0, 16]):
        with pytest.raises(ValueError):
            orc.quantize_grouped(x, off)


# ----------------------------------------------------------------- 2D weight

def test_weight_2d_scale_is_max_of_1d_scales(orc):
    w = inputs.random_shape(10, 64, 96, "wide")
    two = orc.quantize_weight_2d(w)
    one = orc.quantize(w, flags=orc.ROWWISE)
    assert np.array_equal(two["amax_row"], one["amax_row"])
    N, B = one["sf_row"].shape
    band_max = one["sf_row"].reshape(N // 16, 16, B).max(axis=1)
    assert np.array_equal(two["sf_row"], np.repeat(band_max, 16, axis=0))
    # rows whose 1D scale already equals the band's scale encode exactly as in 1D
    same = (one["sf_row"] == two["sf_row"]).repeat(8, axis=1)
    assert np.array_equal(two["q_row"][same], one["q_row"][same])


def test_weight_2d_transposition_invariant_with_equal_amax(orc):
    rng = np.random.default_rng(11)
    n = 64
    w = rng.uniform(-1.0, 1.0, (n, n)).astype(np.float32)
    perm = rng.permutation(n)
    w[np.arange(n), perm] = rng.choice([-1.5, 1.5], n)  # every row and column has amax 1.5
    wb = torch.from_numpy(w).to(torch.bfloat16)
    a = orc.quantize_weight_2d(wb)
    b = orc.quantize_weight_2d(wb.t().contiguous())
    assert (a["amax_row"] == 1.5).all() and (b["amax_row"] == 1.5).all()
    ca = np.empty((n, n), np.uint8)
    ca[:, 0::2], ca[:, 1::2] = a["q_row"] & 0xF, a["q_row"] >> 4
    cb = np.empty((n, n), np.uint8)
    cb[:, 0::2], cb[:, 1::2] = b["q_row"] & 0xF, b["q_row"] >> 4
    assert np.array_equal(ca, cb.T)
    sa = a["sf_row"][::16]  # one row per band: [n/16, n/16] block scales
    sb = b["sf_row"][::16]
    assert np.array_equal(sa, sb.T)


def test_shape_rejections(orc):
    for M, K in [(15, 32), (32, 20), (0, 16)]:
        x = torch.zeros((M, K), dtype=torch.bfloat16)
        with pytest.raises(ValueError):
            orc.quantize(x)
