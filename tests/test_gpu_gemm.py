"""The per-token NVFP4 GEMM (tcgen05 block-scaled MMA) against the oracle's exact sum.

The oracle (oracle_gemm_per_token) sums the exact block products in 128-bit integers and
scales once by the exact product of the two binary32 decode scales; it also returns mag,
the same expression over the products' magnitudes. The kernel accumulates in fp32 in
the tensor cores and rounds twice in the epilogue (times S_dec(a), times S_dec(b)). Each
16-element block product is exact in binary32 (at most 20 significant bits), so if the
hardware rounds at most once per block product it adds, the error is at most
    (K/16 + 2) * 2^-24 * mag        (first order; 2^-20 relative slack for the rest).
Cases whose every partial sum is exact in binary32 (unit scales and decode scales; or
scales in [0.5, 2] with a single 64-element slice of K nonzero) must be bit-exact: they
pin the code layout, the nibble order and the mapping of block scales to rows and K
steps independently of the accumulation order.
"""
import numpy as np
import pytest
import torch

import precision_quantization_row_b200 as nv
from precision_quantization_row_b200 import inputs

pytestmark = pytest.mark.gpu


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_gemm(qa, sfa, aa, qb, sfb, ab):
    ws = nv.new_gemm_workspace(qa.shape[0], qb.shape[0], 2 * qa.shape[1], "cuda")
    d = nv.gemm_per_token(_t(qa), _t(sfa), _t(aa), _t(qb), _t(sfb), _t(ab), workspace=ws)
    assert nv.workspace_error(ws) == 0
    return d.cpu().numpy().astype(np.float64)


def check_bound(got, want, mag, k, label):
    bound = (k / 16 + 2) * 2.0**-24 * mag * (1 + 2.0**-20)
    bad = np.abs(got - want) > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{label}: {int(bad.sum())} of {got.size} outside the bound; first at {tuple(i)}: "
                             f"got {got[tuple(i)]!r} want {want[tuple(i)]!r} bound {bound[tuple(i)]!r}")


def _codes(rng, rows, k):
    return rng.integers(0, 256, (rows, k // 2), dtype=np.uint8)


@pytest.mark.parametrize("mnk", [(128, 256, 256), (256, 512, 512), (48, 80, 768)], ids=lambda s: "x".join(map(str, s)))
def test_exact_unit_scales(orc, mnk):
    """Unit block scales and decode scales (amax = 2688): every partial sum is a multiple of
    1/4 below 2^14, so D is exact whatever the accumulation order."""
    m, n, k = mnk
    rng = np.random.default_rng(m + n + k)
    qa, qb = _codes(rng, m, k), _codes(rng, n, k)
    sfa = np.full((m, k // 16), 0x38, np.uint8)
    sfb = np.full((n, k // 16), 0x38, np.uint8)
    aa = np.full(m, 2688.0, np.float32)
    ab = np.full(n, 2688.0, np.float32)
    want, _ = orc.gemm_per_token(qa, sfa, aa, qb, sfb, ab)
    assert np.array_equal(gpu_gemm(qa, sfa, aa, qb, sfb, ab), want)


@pytest.mark.parametrize("lo", [0, 64, 192, 256, 448], ids=lambda v: f"k{v}")
def test_exact_block_scales_one_mma_step(orc, lo):
    """Scales in [0.5, 2] per (row, block) with only K = lo .. lo+63 nonzero: the one MMA step
    that sees data sums 64 products exactly, so D is exact and any mix-up of block scales
    between rows, blocks or K steps shows."""
    m, n, k = 128, 256, 512
    rng = np.random.default_rng(100 + lo)
    qa, qb = _codes(rng, m, k), _codes(rng, n, k)
    keep = np.zeros(k // 2, bool)
    keep[lo // 2:(lo + 64) // 2] = True
    qa[:, ~keep] = 0
    qb[:, ~keep] = 0
    sfa = rng.integers(0x30, 0x41, (m, k // 16), dtype=np.uint8)
    sfb = rng.integers(0x30, 0x41, (n, k // 16), dtype=np.uint8)
    aa = np.full(m, 2688.0, np.float32)
    ab = np.full(n, 2688.0, np.float32)
    want, _ = orc.gemm_per_token(qa, sfa, aa, qb, sfb, ab)
    assert np.array_equal(gpu_gemm(qa, sfa, aa, qb, sfb, ab), want)


@pytest.mark.parametrize("mnk", [(128, 256, 1024), (256, 512, 4096), (48, 80, 256), (384, 272, 2048),
                                 (16, 16, 256), (144, 528, 768)], ids=lambda s: "x".join(map(str, s)))
def test_general_within_bound(orc, mnk):
    """All block-scale codes (zero and subnormal E4M3 included), random outer amaxes, a zero
    row (amax 0: S_dec = 0), ragged M and N tiles."""
    m, n, k = mnk
    rng = np.random.default_rng(7 * m + n + k)
    qa, qb = _codes(rng, m, k), _codes(rng, n, k)
    sfa = rng.integers(0, 0x7F, (m, k // 16), dtype=np.uint8)
    sfb = rng.integers(0, 0x7F, (n, k // 16), dtype=np.uint8)
    aa = (rng.random(m) * 100).astype(np.float32)
    ab = (rng.random(n) * 100).astype(np.float32)
    aa[min(3, m - 1)] = 0.0
    want, mag = orc.gemm_per_token(qa, sfa, aa, qb, sfb, ab)
    got = gpu_gemm(qa, sfa, aa, qb, sfb, ab)
    check_bound(got, want, mag, k, f"gemm {mnk}")
    assert np.all(got[min(3, m - 1)] == 0.0)


def test_operands_from_the_cast(orc):
    """Activations and weights through the cast's rowwise outputs, then the GEMM."""
    x = inputs.random_shape(31, 512, 2048, "normal").cuda()
    w = inputs.random_shape(32, 768, 2048, "wide").cuda()
    ra = {k: v.cpu().numpy() for k, v in nv.quantize(x, flags=nv.ROWWISE).items()}
    rb = {k: v.cpu().numpy() for k, v in nv.quantize(w, flags=nv.ROWWISE).items()}
    args = (ra["q_row"], ra["sf_row"], ra["amax_row"], rb["q_row"], rb["sf_row"], rb["amax_row"])
    want, mag = orc.gemm_per_token(*args)
    check_bound(gpu_gemm(*args), want, mag, 2048, "cast operands")


@pytest.mark.slow
def test_full_tiling_sampled(orc):
    """4096 x 4096 x 8192 (the full-size tiling: 512 tiles over the grid, 32 pipeline
    stages per tile), compared on 64 sampled rows x 64 sampled columns."""
    m = n = 4096
    k = 8192
    g = torch.Generator(device="cuda").manual_seed(5)
    qa = torch.randint(0, 256, (m, k // 2), dtype=torch.uint8, device="cuda", generator=g)
    qb = torch.randint(0, 256, (n, k // 2), dtype=torch.uint8, device="cuda", generator=g)
    sfa = torch.randint(0, 0x7F, (m, k // 16), dtype=torch.uint8, device="cuda", generator=g)
    sfb = torch.randint(0, 0x7F, (n, k // 16), dtype=torch.uint8, device="cuda", generator=g)
    aa = torch.rand(m, device="cuda", generator=g) * 10
    ab = torch.rand(n, device="cuda", generator=g) * 10
    ws = nv.new_gemm_workspace(m, n, k, "cuda")
    d = nv.gemm_per_token(qa, sfa, aa, qb, sfb, ab, workspace=ws)
    assert nv.workspace_error(ws) == 0
    rng = np.random.default_rng(9)
    rows = np.sort(rng.choice(m, 64, replace=False))
    cols = np.sort(rng.choice(n, 64, replace=False))
    c = lambda t, idx: t.cpu().numpy()[idx]
    want, mag = orc.gemm_per_token(c(qa, rows), c(sfa, rows), c(aa, rows), c(qb, cols), c(sfb, cols), c(ab, cols))
    got = d.cpu().numpy().astype(np.float64)[np.ix_(rows, cols)]
    check_bound(got, want, mag, k, "4096x4096x8192 sampled")


def test_repeated_calls_same_bits():
    """The same call twice writes the same bits (no state survives between calls)."""
    rng = np.random.default_rng(11)
    m, n, k = 256, 256, 1024
    qa, qb = _codes(rng, m, k), _codes(rng, n, k)
    sfa = rng.integers(0, 0x7F, (m, k // 16), dtype=np.uint8)
    sfb = rng.integers(0, 0x7F, (n, k // 16), dtype=np.uint8)
    aa = (rng.random(m) * 5).astype(np.float32)
    ab = (rng.random(n) * 5).astype(np.float32)
    a = gpu_gemm(qa, sfa, aa, qb, sfb, ab)
    b = gpu_gemm(qa, sfa, aa, qb, sfb, ab)
    assert np.array_equal(a.view(np.uint64), b.view(np.uint64))
