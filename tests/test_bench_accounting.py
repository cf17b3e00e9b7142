"""The benchmark's byte accounting (the roofline's numerators) and the keying of the
recorded DRAM traffic, on the CPU."""
import json

import pytest

import bench


@pytest.mark.parametrize("m,k,want", [
    (16384, 8192, 687_964_160),   # the LLM activation: x twice, codes, scales, amax vectors
    (4096, 4096, 86_016_000),     # the dense activation
    (256, 512, 674_816),          # the tiny case
])
def test_compulsory_bytes_of_a_cast(m, k, want):
    assert bench.algo_bytes(m, k) == want


def test_per_kernel_bytes_split_the_cast():
    m, k = 16384, 8192
    row, col = bench.kernel_bytes("rowpass", m, k), bench.kernel_bytes("colpass", m, k)
    assert (row, col) == (344_031_232, 343_965_696)
    # each pass reads x once; the column amax is written by one and read by the other
    assert row + col == bench.algo_bytes(m, k) + 4 * k
    assert bench.kernel_bytes("pass0_zero", m, k) == 4 * k


def test_secondary_op_bytes():
    m, k = 16384, 8192
    rowdata = m * k // 2 + m * k // 16 + 4 * m
    assert bench.op_bytes("dequant", m, k) == rowdata + 2 * m * k == 343_998_464
    assert bench.op_bytes("requant", m, k) == 2 * (m * k // 2 + m * k // 16) + 4 * m + 4 * k


def test_source_hash_ignores_comments_only():
    code = "int f(int a) {\n    return a + 1;   // one more\n}\n/* block\n comment */\n"
    same = "// a header line\nint f(int a)\n{\n  return a + 1;\n}\n"
    other = "int f(int a) { return a + 2; }\n"
    assert bench.kernel_source_sha([code]) == bench.kernel_source_sha([same])
    assert bench.kernel_source_sha([code]) != bench.kernel_source_sha([other])


def test_recorded_traffic_is_used_only_for_the_sources_it_was_taken_on(monkeypatch):
    with open(bench.PROFILE_JSON) as f:
        rec = json.load(f)
    monkeypatch.setattr(bench, "kernel_source_sha", lambda texts=None: rec["kernel_source_sha"])
    for name in ("rowpass", "colpass"):
        k = rec["kernels"][name]
        assert k["dram_bytes_per_launch"] == k["dram_read_bytes"] + k["dram_write_bytes"]
        assert bench.ncu_traffic(name) == k["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "kernel_source_sha", lambda texts=None: "0" * 16)
    assert bench.ncu_traffic("colpass") is None
