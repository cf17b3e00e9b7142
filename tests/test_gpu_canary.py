"""Writes outside the buffers, checked the way a memory sanitizer would (none runs on
the GPU pool): every output, the workspace and the absmax buffers sit between canary
bytes. Each entry point must leave the canaries alone and write the same bytes as the
same call on plain buffers. Shapes cover ragged tails, rows wider than 16384 elements
(the tile path), empty token groups and both unit widths of the dequantization."""
import pytest
import torch

import precision_quantization_row_b200 as nv
from precision_quantization_row_b200 import inputs
from parity_util import canaries_intact, guarded, guarded_outputs

pytestmark = pytest.mark.gpu

OFFSETS = [0, 0, 48, 48, 320, 400]   # five groups over 400 rows, two of them empty


def _bits(t: torch.Tensor) -> torch.Tensor:
    return t.detach().reshape(-1).contiguous().view(torch.uint8).cpu()


def _check(raws, got: dict, want: dict):
    torch.cuda.synchronize()
    assert all(canaries_intact(r) for r in raws), "a write outside a buffer"
    for k in want:
        assert torch.equal(_bits(got[k]), _bits(want[k])), k


@pytest.mark.parametrize("flags", [nv.ROWWISE, nv.COLWISE, nv.ROWWISE | nv.COLWISE], ids=["row", "col", "both"])
@pytest.mark.parametrize("shape", [(16, 16), (48, 80), (272, 144), (1040, 1056), (64, 16400)],
                         ids=lambda s: f"{s[0]}x{s[1]}")
def test_cast(shape, flags):
    rows, cols = shape
    x = inputs.random_shape(80, rows, cols, "normal").cuda()
    raws, out = guarded_outputs(rows, cols, flags, "cuda")
    ws_raw, ws = guarded((nv.workspace_bytes(rows, cols),), torch.uint8, "cuda")
    b_raw, buf = guarded((1,), torch.float32, "cuda")
    buf.fill_(1.5)
    nv.quantize(x, flags=flags, absmax=buf, decay=0.5, out=out, workspace=ws)
    ref_buf = torch.full((1,), 1.5, dtype=torch.float32, device="cuda")
    want = nv.quantize(x, flags=flags, absmax=ref_buf, decay=0.5)
    _check(raws + [ws_raw, b_raw], dict(out, absmax=buf), dict(want, absmax=ref_buf))


def test_grouped_cast():
    rows, cols, G = 400, 272, len(OFFSETS) - 1
    x = inputs.random_shape(81, rows, cols, "wide").cuda()
    raws, out = guarded_outputs(rows, cols, nv.ROWWISE | nv.COLWISE, "cuda", groups=G)
    ws_raw, ws = guarded((nv.workspace_bytes(rows, cols, G),), torch.uint8, "cuda")
    b_raw, bufs = guarded((G,), torch.float32, "cuda")
    bufs.fill_(2.0)
    nv.quantize_grouped(x, OFFSETS, absmax=bufs, decay=0.5, out=out, workspace=ws)
    ref_bufs = torch.full((G,), 2.0, dtype=torch.float32, device="cuda")
    want = nv.quantize_grouped(x, OFFSETS, absmax=ref_bufs, decay=0.5)
    _check(raws + [ws_raw, b_raw], dict(out, absmax=bufs), dict(want, absmax=ref_bufs))


@pytest.mark.parametrize("cols", [272, 16400], ids=["row_pass", "tile_path"])
def test_grouped_cast_noalloc(cols):
    """The entry without allocation: guarded outputs and buffers, the same bytes as the
    workspace entry on plain buffers."""
    rows, G = 400, len(OFFSETS) - 1
    x = inputs.random_shape(85, rows, cols, "wide").cuda()
    raws, out = guarded_outputs(rows, cols, nv.ROWWISE | nv.COLWISE, "cuda", groups=G)
    b_raw, bufs = guarded((G,), torch.float32, "cuda")
    bufs.fill_(2.0)
    nv.quantize_grouped_noalloc(x, OFFSETS, absmax=bufs, decay=0.5, out=out)
    ref_bufs = torch.full((G,), 2.0, dtype=torch.float32, device="cuda")
    want = nv.quantize_grouped(x, OFFSETS, absmax=ref_bufs, decay=0.5)
    _check(raws + [b_raw], dict(out, absmax=bufs), dict(want, absmax=ref_bufs))


@pytest.mark.parametrize("shape", [(144, 272), (64, 16400)], ids=lambda s: f"{s[0]}x{s[1]}")
def test_weight_2d(shape):
    rows, cols = shape
    w = inputs.random_shape(82, rows, cols, "normal").cuda()
    raws, out = guarded_outputs(rows, cols, nv.ROWWISE, "cuda")
    ws_raw, ws = guarded((nv.workspace_bytes(rows, cols),), torch.uint8, "cuda")
    nv.quantize_weight_2d(w, out=out, workspace=ws)
    _check(raws + [ws_raw], out, nv.quantize_weight_2d(w))


# (48, 80): rows of 5 blocks (one block per thread); (272, 1056): 66 blocks (two per thread)
@pytest.mark.parametrize("shape", [(48, 80), (272, 1056)], ids=lambda s: f"{s[0]}x{s[1]}")
def test_dequantize(shape):
    rows, cols = shape
    r = nv.quantize(inputs.random_shape(83, rows, cols, "wide").cuda(), flags=nv.ROWWISE)
    o_raw, out = guarded((rows, cols), torch.bfloat16, "cuda")
    nv.dequantize(r["q_row"], r["sf_row"], r["amax_row"], out=out)
    _check([o_raw], {"x": out}, {"x": nv.dequantize(r["q_row"], r["sf_row"], r["amax_row"])})


@pytest.mark.parametrize("shape,offsets", [((64, 12288), None), ((64, 16400), None), ((400, 272), OFFSETS)],
                         ids=["row_pass", "tile_path", "grouped"])
def test_requantize(shape, offsets):
    rows, cols = shape
    G = 1 if offsets is None else len(offsets) - 1
    r = nv.quantize(inputs.random_shape(84, rows, cols, "normal").cuda(), flags=nv.ROWWISE)
    raws, out = guarded_outputs(rows, cols, nv.COLWISE, "cuda", groups=G)
    ws_raw, ws = guarded((nv.requantize_workspace_bytes(rows, cols, G),), torch.uint8, "cuda")
    b_raw, bufs = guarded((G,), torch.float32, "cuda")
    bufs.fill_(0.25)
    nv.requantize_colwise(r["q_row"], r["sf_row"], r["amax_row"], offsets=offsets, absmax=bufs, decay=0.5,
                          out=out, workspace=ws)
    ref_bufs = torch.full((G,), 0.25, dtype=torch.float32, device="cuda")
    want = nv.requantize_colwise(r["q_row"], r["sf_row"], r["amax_row"], offsets=offsets, absmax=ref_bufs, decay=0.5)
    _check(raws + [ws_raw, b_raw], dict(out, absmax=bufs), dict(want, absmax=ref_bufs))


def test_gemm():
    m, n, k = 144, 272, 512
    g = torch.Generator(device="cuda").manual_seed(86)
    qa = torch.randint(0, 256, (m, k // 2), dtype=torch.uint8, device="cuda", generator=g)
    qb = torch.randint(0, 256, (n, k // 2), dtype=torch.uint8, device="cuda", generator=g)
    sfa = torch.randint(0, 0x7F, (m, k // 16), dtype=torch.uint8, device="cuda", generator=g)
    sfb = torch.randint(0, 0x7F, (n, k // 16), dtype=torch.uint8, device="cuda", generator=g)
    aa = torch.rand(m, device="cuda", generator=g)
    ab = torch.rand(n, device="cuda", generator=g)
    d_raw, d = guarded((m, n), torch.float32, "cuda")
    ws_raw, ws = guarded((nv.gemm_workspace_bytes(m, n, k),), torch.uint8, "cuda")
    nv.gemm_per_token(qa, sfa, aa, qb, sfb, ab, out=d, workspace=ws)
    _check([d_raw, ws_raw], {"d": d}, {"d": nv.gemm_per_token(qa, sfa, aa, qb, sfb, ab)})


def test_update_absmax():
    v = torch.rand(1000, dtype=torch.float32, device="cuda") * 3
    b_raw, buf = guarded((1,), torch.float32, "cuda")
    buf.fill_(1.0)
    nv.update_absmax(buf, v, 0.5)
    ref = torch.ones(1, dtype=torch.float32, device="cuda")
    nv.update_absmax(ref, v, 0.5)
    _check([b_raw], {"b": buf}, {"b": ref})
