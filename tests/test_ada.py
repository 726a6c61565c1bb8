"""Host-side working-rank policy of Ada-Orth-Dion (CPU)."""
import pytest
import torch

from orthonormalized_update_optimizers_b200 import ada


def test_next_rank_follows_the_estimate_within_bounds():
    assert ada.next_rank(10.0, 32, 8, 64) == 13          # ceil(1.25 * 10)
    assert ada.next_rank(100.0, 32, 8, 64) == 64         # clamped above
    assert ada.next_rank(1.0, 32, 8, 64) == 8            # clamped below
    assert ada.next_rank(0.0, 32, 8, 64) == 8            # no signal -> r_min
    assert ada.next_rank(40.0, 32, 8, 64, max_step=4) == 36
    assert ada.next_rank(2.0, 32, 8, 64, max_step=4) == 28
    assert ada.next_rank(20.0, 32, 8, 64, slack=1.0) == 20
    with pytest.raises(ValueError):
        ada.next_rank(5.0, 4, 0, 8)


def test_resize_state_keeps_the_strongest_rows_and_grows_with_fresh_rows():
    n = 40
    Q = torch.linalg.qr(torch.randn(n, 6, generator=torch.Generator().manual_seed(0)))[0].T
    Q = Q.contiguous()
    sigma = [0.5, 3.0, 0.1, 2.0, 1.0, 0.2]
    Q3 = ada.resize_state(Q, sigma, 3)
    assert torch.equal(Q3, Q[[1, 3, 4]])                # largest sigma, original order
    assert torch.allclose(Q3 @ Q3.T, torch.eye(3), atol=1e-6)
    g = torch.Generator().manual_seed(1)
    Q8 = ada.resize_state(Q, sigma, 8, generator=g)
    assert Q8.shape == (8, n) and torch.equal(Q8[:6], Q)
    g2 = torch.Generator().manual_seed(1)
    assert torch.equal(ada.resize_state(Q, sigma, 8, generator=g2), Q8)   # deterministic
    assert ada.resize_state(Q, sigma, 6) is Q
    with pytest.raises(ValueError):
        ada.resize_state(Q, sigma, 0)
    with pytest.raises(ValueError):
        ada.resize_state(Q, sigma[:5], 3)
