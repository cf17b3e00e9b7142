"""The Python binding checks every buffer's dtype, contiguity and size before it calls
the C ABI (which takes raw pointers and cannot see sizes). The checks run in the same
order on CPU tensors, where the call then stops at "must be a CUDA tensor"."""
import pytest
import torch

import precision_quantization_row_b200 as nv
from precision_quantization_row_b200 import build

R, C = 32, 64


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def _x():
    return torch.zeros((R, C), dtype=torch.bfloat16)


def _out(flags=nv.ROWWISE | nv.COLWISE, groups=1):
    return nv._outputs(R, C, flags, "cpu", col_rows=R if groups > 1 else None, groups=groups)


def test_well_formed_cpu_call_stops_at_the_device_check():
    with pytest.raises(TypeError, match="CUDA"):
        nv.quantize(_x(), out=_out(), workspace=nv.new_workspace(R, C), absmax=torch.zeros(1))


@pytest.mark.parametrize("key", ["q_row", "sf_row", "amax_row", "q_col", "sf_col", "amax_col"])
def test_short_output_is_refused(key):
    out = _out()
    out[key] = out[key].reshape(-1)[:-1]
    with pytest.raises(ValueError, match=key):
        nv.quantize(_x(), out=out)


def test_output_of_the_direction_not_asked_for_is_ignored():
    out = _out(nv.ROWWISE)
    with pytest.raises(TypeError, match="CUDA"):
        nv.quantize(_x(), flags=nv.ROWWISE, out=out)


def test_wrong_dtype_and_layout_are_refused():
    out = _out()
    out["amax_row"] = out["amax_row"].double()
    with pytest.raises(TypeError, match="amax_row"):
        nv.quantize(_x(), out=out)
    out = _out()
    out["q_col"] = torch.zeros((R // 2 * 2, C), dtype=torch.uint8).t()   # right size, not contiguous
    with pytest.raises(ValueError, match="contiguous"):
        nv.quantize(_x(), out=out)
    with pytest.raises(TypeError):
        nv.quantize(torch.zeros((R, C), dtype=torch.float16))
    with pytest.raises(TypeError, match="absmax"):
        nv.quantize(_x(), out=_out(), absmax=torch.zeros(1, dtype=torch.float64))


def test_short_workspace_is_refused():
    ws = nv.new_workspace(R, C)[:-1]
    with pytest.raises(ValueError, match="workspace"):
        nv.quantize(_x(), out=_out(), workspace=ws)
    with pytest.raises(ValueError, match="workspace"):
        nv.quantize_weight_2d(_x(), out=_out(nv.ROWWISE), workspace=ws)


def test_grouped_sizes():
    offs = [0, 16, 32]
    out = _out(groups=2)
    with pytest.raises(ValueError, match="absmax"):
        nv.quantize_grouped(_x(), offs, out=out, absmax=torch.zeros(1))    # one buffer per group
    out["amax_col"] = torch.zeros(C)                                        # [G, cols] needed
    with pytest.raises(ValueError, match="amax_col"):
        nv.quantize_grouped(_x(), offs, out=out)
    with pytest.raises(TypeError, match="CUDA"):
        nv.quantize_grouped(_x(), offs, out=_out(groups=2), absmax=torch.zeros(2))


def test_dequantize_and_requantize_inputs():
    q = torch.zeros((R, C // 2), dtype=torch.uint8)
    sf = torch.zeros((R, C // 16), dtype=torch.uint8)
    a = torch.zeros(R)
    with pytest.raises(ValueError, match="sf"):
        nv.dequantize(q, sf[:-1], a)
    with pytest.raises(ValueError, match="amax"):
        nv.dequantize(q, sf, a[:-1])
    with pytest.raises(TypeError, match="out"):
        nv.dequantize(q, sf, a, out=torch.zeros((R, C), dtype=torch.float32))
    with pytest.raises(TypeError, match="CUDA"):
        nv.dequantize(q, sf, a)
    with pytest.raises(ValueError, match="sf_row"):
        nv.requantize_colwise(q, sf[:-1], a)
    with pytest.raises(ValueError, match="absmax"):
        nv.requantize_colwise(q, sf, a, offsets=[0, 16, 32], absmax=torch.zeros(1))
    with pytest.raises(ValueError, match="workspace"):
        nv.requantize_colwise(q, sf, a, workspace=torch.zeros(8, dtype=torch.uint8))
    with pytest.raises(TypeError, match="CUDA"):
        nv.requantize_colwise(q, sf, a)


def test_absmax_update_and_error_word():
    with pytest.raises(TypeError, match="amax_vec"):
        nv.update_absmax(torch.zeros(1), torch.zeros(4, dtype=torch.float16), 0.5)
    with pytest.raises(ValueError, match="absmax"):
        nv.update_absmax(torch.zeros(0), torch.zeros(4), 0.5)
    with pytest.raises(TypeError, match="CUDA"):
        nv.update_absmax(torch.zeros(1), torch.zeros(4), 0.5)
    with pytest.raises(ValueError, match="workspace"):
        nv.workspace_error(torch.zeros(2, dtype=torch.uint8))
