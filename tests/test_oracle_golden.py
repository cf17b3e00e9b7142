"""The oracle against hand-worked blocks (tests/golden/hand_blocks.json).

Each expected byte there was derived by hand from the definition; the file shows
the arithmetic. These pin the block arithmetic: the order RN(RN(ba/6)*s_enc),
s_enc = 2688/amax, enc = s_enc/float(sf), E4M3 and E2M1 ties, saturation, the
sign of zero, the nibble order, and the row/column layouts.
"""
import json
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_blocks.json")


def _load():
    with open(GOLDEN) as f:
        return json.load(f)


def _matrix(case):
    M, K = case["shape"]
    x = np.zeros((M, K), np.float32)
    for r, vals in case["rows"].items():
        x[int(r)] = [float(v) for v in vals]  # "-0" parses to -0.0
    t = torch.from_numpy(x).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.from_numpy(x)), "hand-worked inputs must be exact in bf16"
    return t


def _hex(s):
    return np.array([int(b, 16) for b in s.split()], np.uint8)


@pytest.mark.parametrize("case", _load()["cases"], ids=lambda c: c["name"])
def test_hand_worked_block(orc, case):
    x = _matrix(case)
    out = orc.quantize(x)
    exp = case["expect"]
    for r, v in exp.get("amax_row", {}).items():
        assert out["amax_row"][int(r)] == np.float32(v)
    for r, v in exp.get("sf_row", {}).items():
        assert np.array_equal(out["sf_row"][int(r)], _hex(v)), (r, out["sf_row"][int(r)])
    for r, v in exp.get("q_row", {}).items():
        assert np.array_equal(out["q_row"][int(r)], _hex(v)), (r, out["q_row"][int(r)])
    for c, v in exp.get("amax_col", {}).items():
        assert out["amax_col"][int(c)] == np.float32(v)
    for c, v in exp.get("sf_col", {}).items():
        assert np.array_equal(out["sf_col"][int(c)], _hex(v)), (c, out["sf_col"][int(c)])
    for c, v in exp.get("q_col", {}).items():
        assert np.array_equal(out["q_col"][int(c)], _hex(v)), (c, out["q_col"][int(c)])


def test_hand_worked_intermediates(orc):
    """The intermediate values of case A and C, block by block."""
    assert orc.s_enc(6.0) == 448.0 and orc.s_enc(10.5) == 256.0 and orc.s_enc(2688.0) == 1.0
    assert orc.s_enc(0.0) == 1.0
    u = orc.block_scale_arg(2.0, 448.0)
    assert u == 9786710 * 2.0 ** -16
    assert orc.e4m3(u) == 0x71 and orc.e4m3_decode(0x71) == 144.0
    assert orc.block_enc(0x71, 448.0) == 13048946 * 2.0 ** -22
    assert orc.block_scale_arg(6.375 / 256, 256.0) == 1.0625 and orc.e4m3(1.0625) == 0x38
    assert orc.block_scale_arg(7.125 / 256, 256.0) == 1.1875 and orc.e4m3(1.1875) == 0x3A
    assert orc.block_enc(0x3A, 256.0) == 13421773 * 2.0 ** -16
    assert orc.block_enc(0, 448.0) == 0.0


@pytest.mark.parametrize("seq", _load()["absmax_sequences"]["cases"])
def test_absmax_sequences(orc, seq):
    buf = seq["start"]
    for obs, want in zip(seq["observed"], seq["expect"]):
        buf = orc.update_absmax(buf, [obs * 0.5, obs, 0.0], seq["decay"])
        assert buf == want
