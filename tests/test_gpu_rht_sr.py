"""The cast with the columnwise options (nvfp4pt_quantize_grouped_opts) against the oracle,
bit-exact: the Hadamard transform of each columnwise 16-row block, stochastic rounding
with Philox words, and both; ungrouped and grouped (empty and ragged groups), tasks
that end inside a 512-row task, column strips with a partial quad. The rowwise outputs
and the running buffers must be those of the plain cast (the row direction never uses
the options)."""
import numpy as np
import pytest
import torch

import precision_quantization_row_b200 as nv
from precision_quantization_row_b200 import inputs
from parity_util import compare, oracle_colwise_opts_parallel, oracle_quantize_parallel, to_np

pytestmark = pytest.mark.gpu
RC = nv.ROWWISE | nv.COLWISE
SIGNS = 0b1011_0110_0101_1100

MODES = {"rht": dict(rht=True, rht_signs=SIGNS), "sr": dict(sr=True, seed=0x1234_5678_9ABC_DEF0, offset=7),
         "rht_sr": dict(rht=True, rht_signs=0x5A3C, sr=True, seed=3, offset=(5 << 32) | 9)}
SHAPES = [(256, 512, None), (96, 48, None), (544, 80, None), (400, 272, [0, 16, 48, 48, 400]),
          (1040, 1056, [0, 128, 512, 512, 1040])]


def _gpu(x, offsets, decay=0.5, **opts):
    G = 1 if offsets is None else len(offsets) - 1
    bufs = torch.full((G,), 2.0, dtype=torch.float32, device="cuda")
    ws = nv.new_workspace(*x.shape, G, device="cuda")
    out = to_np(nv.quantize_grouped_opts(x.cuda(), offsets, absmax=bufs, decay=decay, workspace=ws, **opts))
    assert nv.workspace_error(ws) == 0
    out["absmax"] = bufs.cpu().numpy()
    return out


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}x{s[1]}{'g' if s[2] else ''}")
def test_options_match_oracle(orc, mode, shape):
    rows, cols, offsets = shape
    x = inputs.random_shape(rows + cols, rows, cols, "wide")
    got = _gpu(x, offsets, **MODES[mode])
    want_col = orc.quantize_colwise_opts(x, offsets=offsets, **MODES[mode])
    compare(got, want_col, label=f"{mode} {shape} colwise")
    G = 1 if offsets is None else len(offsets) - 1
    plain = orc.quantize_grouped(x, [0, rows] if offsets is None else offsets,
                                 absmax=np.full(G, 2.0, np.float32), decay=0.5)
    compare(got, {k: plain[k] for k in ("q_row", "sf_row", "amax_row", "absmax")}, label=f"{mode} {shape} rowwise")


def test_no_options_is_the_plain_cast():
    x = inputs.random_shape(61, 400, 272, "normal").cuda()
    offsets = [0, 16, 48, 48, 400]
    a = nv.quantize_grouped_opts(x, offsets)
    b = nv.quantize_grouped(x, offsets)
    for k in b:
        assert torch.equal(a[k].view(torch.uint8), b[k].view(torch.uint8)), k


def test_sr_words_follow_seed_and_offset():
    x = inputs.random_shape(62, 256, 128, "normal").cuda()
    a = nv.quantize_grouped_opts(x, sr=True, seed=1, offset=0)
    b = nv.quantize_grouped_opts(x, sr=True, seed=1, offset=0)
    c = nv.quantize_grouped_opts(x, sr=True, seed=1, offset=1)
    d = nv.quantize_grouped_opts(x, sr=True, seed=2, offset=0)
    assert torch.equal(a["q_col"], b["q_col"])
    assert not torch.equal(a["q_col"], c["q_col"])
    assert not torch.equal(a["q_col"], d["q_col"])
    assert torch.equal(a["sf_col"], c["sf_col"])


@pytest.mark.slow
def test_options_headline_full_size(orc):
    """The 16384 x 8192 activation with the transform and stochastic rounding."""
    x = inputs.llm()
    opts = MODES["rht_sr"]
    got = to_np(nv.quantize_grouped_opts(x.cuda(), **opts))
    compare(got, oracle_colwise_opts_parallel(x, **opts), label="llm rht+sr colwise")
    compare(got, {k: v for k, v in oracle_quantize_parallel(x, flags=nv.ROWWISE).items()}, label="llm rowwise")


@pytest.mark.slow
def test_options_moe_full_size(orc):
    """The grouped MoE workload with the transform (64 token groups)."""
    x, offsets = inputs.moe()
    got = to_np(nv.quantize_grouped_opts(x.cuda(), offsets, rht=True, rht_signs=SIGNS))
    want = oracle_colwise_opts_parallel(x, offsets=offsets, rht=True, rht_signs=SIGNS)
    compare({k: got[k] for k in want}, want, label="moe rht colwise")
