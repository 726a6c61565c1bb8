"""Per-layer working-rank policy for Ada-Orth-Dion.

"Orth-Dion: Eliminating Geometric Mismatch in Distributed Low-Rank Spectral
Optimization", Ada-Orth-Dion, gives the mechanism but not the formulas:
every layer's working rank follows an entropy-based estimate of the
intrinsic dimensionality of its gradient spectrum, taken from the power
iteration's factors, so that the rank sits at the layer's signal-to-noise
transition and the QR step costs less (Key Results: the average working
rank fell to about 93% of the fixed rank).  The readings taken here:

* the estimate is the effective rank of the power iteration's singular-value
  estimates: dion_lowrank_step(..., sigma=...) writes sigma_j = ||R_j||, and
  dion_effective_rank turns them into exp(H(sigma^2 / sum sigma^2));
* the next rank is ceil(slack * estimate), clamped to [r_min, r_max] and
  moved by at most max_step per step;
* the state follows the rank: a shrinking Q_state keeps its rows with the
  largest sigma (in their order), a growing one gains rows drawn
  N(0, 1/n); the next step's power iteration orthonormalizes P = orth(B Q)
  either way.

The library steps matrices of different ranks in one call (params.rank = 0
takes each matrix's rank from its Q_state rows).  This module is host-side
policy only.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import torch


def next_rank(erank: float, r: int, r_min: int, r_max: int, slack: float = 1.25,
              max_step: Optional[int] = None) -> int:
    """The working rank for the next step from this step's estimate."""
    if not (1 <= r_min <= r_max):
        raise ValueError("need 1 <= r_min <= r_max")
    target = math.ceil(slack * float(erank)) if erank > 0 else r_min
    target = max(r_min, min(r_max, target))
    if max_step is not None:
        target = max(r - max_step, min(r + max_step, target))
        target = max(r_min, min(r_max, target))
    return int(target)


def resize_state(Qt: torch.Tensor, sigma: Sequence[float], r_new: int,
                 generator: Optional[torch.Generator] = None) -> torch.Tensor:
    """Q_state (r x n, rows = the columns of Q) resized to r_new rows: the
    rows with the largest sigma are kept in their order when shrinking, and
    rows drawn N(0, 1/n) are appended when growing.  Returns a new
    contiguous tensor (the same one if r_new == r)."""
    r, n = Qt.shape
    if r_new < 1 or r_new > n:
        raise ValueError("r_new outside [1, n]")
    if len(sigma) != r:
        raise ValueError("sigma needs one value per row")
    if r_new == r:
        return Qt
    if r_new < r:
        order = sorted(range(r), key=lambda j: (-float(sigma[j]), j))[:r_new]
        keep = torch.tensor(sorted(order), dtype=torch.long, device=Qt.device)
        return Qt.index_select(0, keep).contiguous()
    extra = torch.randn((r_new - r, n), generator=generator, dtype=torch.float32,
                        device="cpu" if generator is None else generator.device)
    extra = (extra / math.sqrt(n)).to(device=Qt.device, dtype=Qt.dtype)
    return torch.cat([Qt, extra], dim=0).contiguous()
