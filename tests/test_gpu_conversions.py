"""The device conversions the cast kernels use, over their whole input domains,
against the CPU definition (the oracle's table conversions, themselves pinned to
the OCP formats and to ml_dtypes/torch in test_oracle_tables.py).

* Every binary32 pattern from +0 to +inf and from -0 to -inf goes through the
  device E2M1 and E4M3 conversions; the device reports where the code changes.
  The oracle is monotone in |v|, so checking it at both ends of every constant
  interval of the device function proves they agree on all 2^32 - 2^24 inputs.
* The operand order of the packed conversions (low nibble / low byte first).
* The E4M3 decode of every code in both byte positions.
* The division of every finite non-negative bf16 block amax by 6.
"""
import ctypes

import numpy as np
import pytest
import torch

import probe

pytestmark = pytest.mark.gpu

RANGES = [(0x00000000, 0x7F800000), (0x80000000, 0xFF800000)]


def _transitions(which: int):
    cap = 1 << 16
    out = torch.zeros(2 * cap, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = probe.lib().nvfp4pt_probe_transitions(which, ctypes.c_void_p(out.data_ptr()), cap,
                                            ctypes.c_void_p(cnt.data_ptr()),
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    n = int(cnt.item())
    assert 0 < n <= cap
    rec = out[: 2 * n].cpu().numpy().view(np.uint32).reshape(n, 2)
    return rec[np.argsort(rec[:, 0])]


def _check_against_oracle(rec, conv):
    for lo, hi in RANGES:
        r = rec[(rec[:, 0] >= lo) & (rec[:, 0] <= hi)]
        assert r[0, 0] == lo
        starts = r[:, 0].astype(np.int64)
        ends = np.append(starts[1:] - 1, hi)
        a = conv(starts.astype(np.uint32).view(np.float32))
        b = conv(ends.astype(np.uint32).view(np.float32))
        assert np.array_equal(a, r[:, 1]), "interval starts"
        assert np.array_equal(b, r[:, 1]), "interval ends"


def test_e2m1_device_conversion_exhaustive(orc):
    rec = _transitions(0)
    assert rec.shape[0] == 16  # 8 codes per sign
    _check_against_oracle(rec, orc.e2m1_array)


def test_e4m3_device_conversion_exhaustive(orc):
    rec = _transitions(1)
    assert rec.shape[0] == 2 * 127  # 0x00..0x7E per sign
    _check_against_oracle(rec, orc.e4m3_array)


def _pairs(lo_hi):
    a = torch.tensor(np.asarray(lo_hi, np.float32).ravel(), device="cuda")
    n = a.numel() // 2
    out = torch.zeros(n, dtype=torch.int32, device="cuda")
    st = probe.lib().nvfp4pt_probe_pairs(ctypes.c_void_p(a.data_ptr()), n, ctypes.c_void_p(out.data_ptr()),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    return out.cpu().numpy().view(np.uint32)


def test_pair_order(orc):
    w = _pairs([[0.5, 6.0], [1.0, 448.0], [-0.0, 0.0], [3.0, -1.0]])
    assert w[0] & 0xFF == 0x71                 # 0.5 -> 1 low nibble, 6 -> 7 high nibble
    assert (w[1] >> 16) == (0x7E << 8 | 0x38)  # 1.0 -> 0x38 low byte, 448 -> 0x7E high byte
    assert w[2] & 0xFF == 0x08                 # -0.0 keeps its sign
    assert w[3] & 0xFF == 0xA5                 # 3 -> 5, -1 -> 0xA
    rng = np.random.default_rng(0)
    v = (rng.standard_normal((4096, 2)) * np.exp2(rng.uniform(-12, 10, (4096, 2)))).astype(np.float32)
    w = _pairs(v)
    lo, hi = v[:, 0], v[:, 1]
    assert np.array_equal(w & 0xF, orc.e2m1_array(lo))
    assert np.array_equal((w >> 4) & 0xF, orc.e2m1_array(hi))
    ok = (np.abs(lo) <= 448) & (np.abs(hi) <= 448)
    assert np.array_equal(((w >> 16) & 0xFF)[ok], orc.e4m3_array(lo[ok]))
    assert np.array_equal((w >> 24)[ok], orc.e4m3_array(hi[ok]))


def test_e4m3_decode(orc):
    out = torch.zeros(512, dtype=torch.float32, device="cuda")
    st = probe.lib().nvfp4pt_probe_e4m3_decode(ctypes.c_void_p(out.data_ptr()),
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    d = out.cpu().numpy()
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue
        want = np.float32(orc.e4m3_decode(c))
        assert d[c].view(np.uint32) == want.view(np.uint32), hex(c)
        assert d[256 + c].view(np.uint32) == want.view(np.uint32), hex(c)


def test_div6_exhaustive():
    out = torch.zeros(0x7F80, dtype=torch.float32, device="cuda")
    st = probe.lib().nvfp4pt_probe_div6(ctypes.c_void_p(out.data_ptr()),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    got = out.cpu().numpy().view(np.uint32)
    b = (np.arange(0x7F80, dtype=np.uint32) << 16).view(np.float32)
    want = (b / np.float32(6.0)).astype(np.float32).view(np.uint32)  # IEEE binary32 division
    assert np.array_equal(got, want)


@pytest.mark.parametrize("lo,hi", [(10, 24), (125, 129), (252, 254)])
def test_block_scale_division_matches_ieee(lo, hi):
    """enc = s_enc / float(sf) as the cast computes it, against the IEEE division, for all
    126 positive E4M3 divisors and every significand of s in the given binades: the low
    binades (down to the smallest possible s_enc, 2688/FLT_MAX ~ 2^-117, where the
    remainder can be subnormal), the middle, and the overflow edge (clamped to FLT_MAX)."""
    bad = torch.zeros(1, dtype=torch.int64, device="cuda")
    st = probe.lib().nvfp4pt_probe_e4m3_div(lo, hi, ctypes.c_void_p(bad.data_ptr()),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    assert int(bad.item()) == 0


def test_packed_block_scales_match_scalar():
    """The block-scale step in the packed two-lane form the column pass uses equals the
    scalar form (pinned to the oracle by the parity tests) bit for bit: every bf16
    block amax, against every 4093rd significand of s in every binade that s_enc can
    take (2688 / max bf16 ~ 2^-117 up to FLT_MAX), plus s = FLT_MAX and s = 1."""
    bad = torch.zeros(1, dtype=torch.int64, device="cuda")
    st = probe.lib().nvfp4pt_probe_pair_scales(10, 254, 4093, ctypes.c_void_p(bad.data_ptr()),
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    assert int(bad.item()) == 0
