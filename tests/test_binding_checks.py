"""CPU checks of the binding's host-side argument checks: device buffers of
the wrong dtype, too short, strided or on the host are refused before any
pointer reaches the library."""
import pytest
import torch

import orthonormalized_update_optimizers_b200 as ouo


def test_check_vector_accepts_none():
    ouo.check_vector(None, "status", torch.int32, 1)


@pytest.mark.parametrize("t,exc,msg", [
    (torch.zeros(4, dtype=torch.float32), TypeError, "must be torch.float64"),
    (torch.zeros(3, dtype=torch.float64), ValueError, "at least 4 elements"),
    (torch.zeros(8, dtype=torch.float64)[::2], ValueError, "contiguous"),
    (torch.zeros(4, dtype=torch.float64), ValueError, "CUDA tensor"),
])
def test_check_vector_refuses(t, exc, msg):
    with pytest.raises(exc, match=msg):
        ouo.check_vector(t, "row_sqnorm", torch.float64, 4)


def test_matrices_must_be_cuda_tensors():
    with pytest.raises(ValueError, match="CUDA tensor"):
        ouo.MatBatch([torch.zeros(4, 4)])
    with pytest.raises(ValueError, match="unit column stride"):
        ouo.MatBatch([torch.zeros(4, 4).t()])


def test_select_rows_requires_its_outputs():
    with pytest.raises(ValueError, match="required"):
        ouo.dion3_select_rows([], None, 0.125, None, [], None)


def test_scale_needs_one_value_per_matrix():
    with pytest.raises(ValueError, match="one value per matrix"):
        ouo.apply_update([], [], 0.02, scale=[1.0])
