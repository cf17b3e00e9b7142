"""The canary helper of the GPU tests, checked on the CPU: the guarded view has the
asked shape, dtype, contiguity and alignment, writes inside it leave the canaries
alone, and a write one byte outside it is seen."""
import pytest
import torch

from parity_util import GUARD, canaries_intact, guarded, guarded_outputs


@pytest.mark.parametrize("shape,dtype", [((48, 40), torch.uint8), ((7,), torch.float32), ((16, 80), torch.bfloat16)])
def test_guarded_view(shape, dtype):
    raw, v = guarded(shape, dtype, "cpu")
    assert v.shape == shape and v.dtype == dtype and v.is_contiguous()
    assert (v.data_ptr() - raw.data_ptr()) == GUARD
    v.fill_(1)
    assert canaries_intact(raw)


@pytest.mark.parametrize("where", [GUARD - 1, -GUARD])
def test_a_write_just_outside_is_seen(where):
    raw, v = guarded((16, 16), torch.uint8, "cpu")
    raw[where] = 0
    assert not canaries_intact(raw)


def test_guarded_outputs_match_the_binding_shapes():
    import precision_quantization_row_b200 as nv
    for groups in (1, 3):
        raws, out = guarded_outputs(48, 80, nv.ROWWISE | nv.COLWISE, "cpu", groups=groups)
        ref = nv._outputs(48, 80, nv.ROWWISE | nv.COLWISE, "cpu", col_rows=48 if groups > 1 else None, groups=groups)
        assert sorted(out) == sorted(ref) and len(raws) == len(out)
        for k in ref:
            assert out[k].shape == ref[k].shape and out[k].dtype == ref[k].dtype, k
