"""GPU parity of the dequantization and the columnwise requantization against the
oracle, bit for bit."""
import numpy as np
import pytest
import torch

import precision_quantization_row_b200 as nv
from precision_quantization_row_b200 import inputs
from parity_util import compare, oracle_quantize_parallel, to_np

pytestmark = pytest.mark.gpu

FINITE_SF = [c for c in range(256) if c not in (0x7F, 0xFF)]


def _random_rows(seed, rows, cols):
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 256, (rows, cols // 2), dtype=np.uint8)
    sf = rng.choice(FINITE_SF, (rows, cols // 16)).astype(np.uint8)
    amax = (rng.standard_normal(rows) * 10.0 ** rng.integers(-30, 30, rows)).astype(np.float32)
    amax = np.abs(amax)
    special = np.array([0.0, 2688.0, 2688.0 * 2 ** -20, 2688.0 * 2 ** 40, 3.3e38, 1e-38, 5e-39, 1.0], np.float32)
    amax[: min(rows, special.size)] = special[: min(rows, special.size)]
    return q, sf, amax


@pytest.mark.parametrize("shape", [(16, 16), (48, 80), (272, 144), (1040, 1056), (4096, 16), (16, 4096)],
                         ids=lambda s: f"{s[0]}x{s[1]}")
def test_dequant_random_codes(orc, shape):
    q, sf, amax = _random_rows(sum(shape), *shape)
    got = nv.dequantize(torch.from_numpy(q).cuda(), torch.from_numpy(sf).cuda(), torch.from_numpy(amax).cuda())
    want = orc.dequantize(q, sf, amax)
    g = got.cpu().view(torch.int16).numpy().view(np.uint16)
    bad = np.argwhere(g != want)
    assert bad.size == 0, f"{bad.shape[0]} mismatches, first {bad[:3].tolist()}"


def test_dequant_overflows_to_infinity(orc):
    """Row amaxes up to the largest binary32: products at or past halfway from the largest
    finite bf16 to 2^128 round to infinity, below it to the largest finite bf16."""
    rng = np.random.default_rng(68)
    rows, cols = 64, 128
    q = rng.integers(0, 256, (rows, cols // 2), dtype=np.uint8)
    sf = rng.choice([0x7E, 0x7D, 0x76, 0x70, 0xFE], (rows, cols // 16)).astype(np.uint8)
    amax = np.linspace(3.0e38, np.finfo(np.float32).max, rows).astype(np.float32)
    want = orc.dequantize(q, sf, amax)
    assert (want & 0x7FFF == 0x7F80).any() and (want & 0x7FFF == 0x7F7F).any()
    got = nv.dequantize(torch.from_numpy(q).cuda(), torch.from_numpy(sf).cuda(), torch.from_numpy(amax).cuda())
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), want)


@pytest.mark.parametrize("shape", [(272, 1056), (48, 80)], ids=lambda s: f"{s[0]}x{s[1]}")
def test_dequant_output_16_byte_aligned(orc, shape):
    """An output 16 bytes past a 32-byte boundary: each block goes out as two 16-byte
    stores (rows with an even and an odd number of blocks)."""
    q, sf, amax = _random_rows(70, *shape)
    rows, cols = shape
    buf = torch.empty(rows * cols + 8, dtype=torch.bfloat16, device="cuda")
    out = buf[8:].view(rows, cols)
    assert out.data_ptr() % 32 == 16
    nv.dequantize(torch.from_numpy(q).cuda(), torch.from_numpy(sf).cuda(), torch.from_numpy(amax).cuda(), out=out)
    want = orc.dequantize(q, sf, amax)
    assert np.array_equal(out.cpu().view(torch.int16).numpy().view(np.uint16), want)


# more units (two blocks each, then one block each for rows of 1025 blocks) than the
# grid's threads at 128 CTAs per SM: threads take several units
@pytest.mark.parametrize("shape", [(10240, 16384), (6144, 16400)], ids=lambda s: f"{s[0]}x{s[1]}")
def test_dequant_grid_stride(orc, shape):
    q, sf, amax = _random_rows(sum(shape), *shape)
    got = nv.dequantize(torch.from_numpy(q).cuda(), torch.from_numpy(sf).cuda(), torch.from_numpy(amax).cuda())
    want = orc.dequantize(q, sf, amax)
    g = got.cpu().view(torch.int16).numpy().view(np.uint16)
    bad = np.argwhere(g != want)
    assert bad.size == 0, f"{bad.shape[0]} mismatches, first {bad[:3].tolist()}"


@pytest.mark.parametrize("kind", ["normal", "wide", "tiny", "signed_zero"])
def test_dequant_of_cast_outputs(orc, kind):
    x = inputs.random_shape(61, 512, 768, kind).cuda()
    out = nv.quantize(x, flags=nv.ROWWISE)
    got = nv.dequantize(out["q_row"], out["sf_row"], out["amax_row"])
    want = orc.dequantize(out["q_row"].cpu().numpy(), out["sf_row"].cpu().numpy(), out["amax_row"].cpu().numpy())
    assert np.array_equal(got.cpu().view(torch.int16).numpy().view(np.uint16), want)


def _rows_of(x):
    out = nv.quantize(x.cuda(), flags=nv.ROWWISE)
    return out["q_row"], out["sf_row"], out["amax_row"]


# (48, 80): a 64-column strip with a partial 8-column group and a 16-row step;
# (64, 16400): rows wider than the cast's row pass takes
@pytest.mark.parametrize("shape", [(256, 512), (1040, 1056), (4096, 4096), (48, 80), (64, 12288), (64, 16400)],
                         ids=lambda s: f"{s[0]}x{s[1]}")
def test_requant_colwise(orc, shape):
    x = inputs.random_shape(62, *shape, "wide")
    q, sf, a = _rows_of(x)
    buf = torch.full((1,), 5.0, device="cuda")
    got = nv.requantize_colwise(q, sf, a, absmax=buf, decay=0.75)
    want = orc.requantize_colwise(q.cpu().numpy(), sf.cpu().numpy(), a.cpu().numpy(),
                                  absmax=np.array([5.0], np.float32), decay=0.75)
    compare(to_np(got), {k: want[k] for k in ("q_col", "sf_col", "amax_col")}, label=f"requant {shape}")
    assert np.float32(buf.item()).view(np.uint32) == np.float32(want["absmax"][0]).view(np.uint32)


def test_requant_grouped(orc):
    x = inputs.random_shape(63, 400, 272, "normal")
    offsets = [0, 0, 48, 48, 320, 400]
    q, sf, a = _rows_of(x)
    bufs = torch.arange(5, dtype=torch.float32, device="cuda")
    got = nv.requantize_colwise(q, sf, a, offsets=offsets, absmax=bufs, decay=0.5)
    want = orc.requantize_colwise(q.cpu().numpy(), sf.cpu().numpy(), a.cpu().numpy(), offsets=offsets,
                                  absmax=np.arange(5, dtype=np.float32), decay=0.5)
    compare(to_np(got), {k: want[k] for k in ("q_col", "sf_col", "amax_col")}, label="grouped requant")
    assert np.array_equal(bufs.cpu().numpy().view(np.uint32), want["absmax"].view(np.uint32))


def test_requant_grouped_wide_rows(orc):
    """Grouped requantization of rows 12288 wide."""
    x = inputs.random_shape(65, 128, 12288, "normal")
    offsets = [0, 64, 64, 128]
    q, sf, a = _rows_of(x)
    got = nv.requantize_colwise(q, sf, a, offsets=offsets)
    want = orc.requantize_colwise(q.cpu().numpy(), sf.cpu().numpy(), a.cpu().numpy(), offsets=offsets)
    compare(to_np(got), {k: want[k] for k in ("q_col", "sf_col", "amax_col")}, label="grouped requant wide")


# widths that are multiples of 256 take the TMA-fed tile kernels, the others the direct ones
@pytest.mark.parametrize("shape,offsets", [((48, 80), None), ((272, 144), None), ((96, 4112), None),
                                          ((400, 272), [0, 16, 16, 240, 400]), ((528, 336), [0, 0, 512, 528]),
                                          ((304, 512), None), ((400, 768), [0, 16, 16, 240, 400]),
                                          ((176, 1280), [0, 0, 48, 112, 176, 176])],
                         ids=["48x80", "272x144", "96x4112", "400x272g", "528x336g", "304x512", "400x768g",
                              "176x1280g"])
def test_requant_random_codes(orc, shape, offsets):
    """Arbitrary codes, every finite block-scale code (negative and subnormal ones too) and
    extreme row amaxes: the requantization is the oracle's columnwise cast of the oracle's
    dequantization, codes, scales, column amaxes and running buffers."""
    q, sf, amax = _random_rows(sum(shape) + 7, *shape)
    G = 1 if offsets is None else len(offsets) - 1
    bufs = torch.linspace(0.5, 4.0, G, dtype=torch.float32, device="cuda")
    want = orc.requantize_colwise(q, sf, amax, offsets=offsets, absmax=bufs.cpu().numpy(), decay=0.5)
    got = nv.requantize_colwise(torch.from_numpy(q).cuda(), torch.from_numpy(sf).cuda(),
                                torch.from_numpy(amax).cuda(), offsets=offsets, absmax=bufs, decay=0.5)
    compare(to_np(got), {k: want[k] for k in ("q_col", "sf_col", "amax_col")}, label=f"requant random {shape}")
    assert np.array_equal(bufs.cpu().numpy().view(np.uint32), want["absmax"].view(np.uint32))


@pytest.mark.parametrize("cols", [64, 256])
def test_requant_many_groups(orc, cols):
    """1024 token groups of 16 rows (and some empty ones): one 16-row step per group."""
    rows = 16 * 1000
    x = inputs.random_shape(66, rows, cols, "normal")
    sizes = [16] * 1000 + [0] * 24
    np.random.default_rng(67).shuffle(sizes)
    offsets = [0] + list(np.cumsum(sizes))
    q, sf, a = _rows_of(x)
    got = nv.requantize_colwise(q, sf, a, offsets=offsets)
    want = orc.requantize_colwise(q.cpu().numpy(), sf.cpu().numpy(), a.cpu().numpy(), offsets=offsets)
    compare(to_np(got), {k: want[k] for k in ("q_col", "sf_col", "amax_col")}, label="requant 1024 groups")


def test_requant_of_lossless_rows_equals_direct_cast():
    """Rows whose cast is lossless: requantizing their rowwise data on the GPU gives the
    GPU's direct columnwise cast of the matrix itself."""
    from test_oracle_dequant import _lossless_matrix
    x = _lossless_matrix(np.random.default_rng(64), 256, 320).cuda()
    q, sf, a = _rows_of(x)
    got = nv.requantize_colwise(q, sf, a)
    direct = nv.quantize(x, flags=nv.COLWISE)
    for k in ("q_col", "sf_col", "amax_col"):
        assert torch.equal(got[k].reshape(-1), direct[k].reshape(-1)), k


@pytest.mark.slow
def test_dequant_and_requant_at_the_benchmark_size(orc):
    """The LLM activation (16384 x 8192) in the launch configuration the benchmark times
    for both ops: the dequantization against the oracle's, and the columnwise
    requantization against the oracle's columnwise cast of the dequantized matrix
    (computed over exact column ranges in parallel)."""
    x = inputs.llm()
    r = nv.quantize(x.cuda(), flags=nv.ROWWISE)
    q, sf, a = (r[k].cpu().numpy() for k in ("q_row", "sf_row", "amax_row"))
    xd = orc.dequantize(q, sf, a)
    got = nv.dequantize(r["q_row"], r["sf_row"], r["amax_row"])
    bad = np.argwhere(got.cpu().view(torch.int16).numpy().view(np.uint16) != xd)
    assert bad.size == 0, f"{bad.shape[0]} mismatches, first {bad[:3].tolist()}"
    del got
    want = oracle_quantize_parallel(torch.from_numpy(xd.view(np.int16)).view(torch.bfloat16), flags=nv.COLWISE)
    got = nv.requantize_colwise(r["q_row"], r["sf_row"], r["amax_row"])
    compare(to_np(got), want, label="requant 16384x8192")
