"""Dion3 row-selection update rule (oracle).

Sources:

* "Dion3: Full-Stack Orthogonal Updates", Abstract: each step orthogonalizes
  only a fraction of the momentum matrix's rows.
* "Dion3：全栈正交更新", 核心模块: a small fraction of rows (e.g. 1/8) is
  orthogonalized per step, the other rows keep the plain momentum update,
  with error feedback; 输入输出流程: momentum -> select rows -> Gram NS ->
  weight update.

Readings (listed in the design notes):

* Selection key: the float64 sum of squares of each row of the updated
  momentum B (fp32-stored).  k = ceil(rho * m) rows with the largest key are
  kept; equal keys go to the lower row index; the kept indices are returned
  in ascending order.
* X0 = B[S] / (||B[S]||_F + eps), eps = 1e-7, with ||B[S]||_F^2 the sum of
  the kept keys.  Newton-Schulz then runs without normalizing again.
* Error feedback (default): B = M + G; kept rows leave mu * B[S] behind in
  the buffer (the orthogonalized share (1 - mu) B[S] is taken out); the
  other rows keep B.  Without error feedback the momentum is the EMA
  M <- mu M + G and selection only reads it.
* The weights change on the kept rows only.

TEST INFRASTRUCTURE: see the package docstring.
"""
from __future__ import annotations

import math

import numpy as np

from . import apply as _apply
from . import momentum as _momentum
from . import ns as _ns

EF_NONE = 0
EF_ROWS = 1


def num_selected(m: int, rho: float) -> int:
    """k = ceil(rho * m), at least 1 and at most m."""
    k = math.ceil(float(rho) * m - 1e-9)
    return max(1, min(m, k))


def select_rows(keys, rho: float) -> np.ndarray:
    """Ascending indices of the k rows with the largest keys (ties: lower
    index first)."""
    keys = np.asarray(keys, dtype=np.float64)
    m = keys.shape[0]
    k = num_selected(m, rho)
    order = np.lexsort((np.arange(m), -keys))  # primary: key desc; then index asc
    return np.sort(order[:k]).astype(np.int32)


def gather_normalize(B, idx, keys, eps: float = _ns.DEFAULT_EPS):
    """X0 = B[idx] / (sqrt(sum keys[idx]) + eps); returns (X0, factor)."""
    B64 = np.asarray(B, dtype=np.float64)
    fro = math.sqrt(float(np.sum(np.asarray(keys, dtype=np.float64)[idx])))
    factor = 1.0 / (fro + eps)
    return B64[idx] * factor, factor


def ef_write(B, idx, mu: float, state_dtype=np.float32):
    """Momentum after error feedback: mu * B on the kept rows, B elsewhere."""
    out = np.asarray(B, dtype=np.float64).copy()
    out[idx] = float(np.float32(mu)) * out[idx]
    return out.astype(state_dtype) if state_dtype is not None else out


def dion3_step(M, G, W, mu: float, rho: float, lr: float, scale: float,
               ef_mode: int = EF_ROWS, iters: int = 5,
               coeffs=_ns.MUON_COEFFS, safety=1, restart_after=(3,),
               wd: float = 0.0, variant: str = "gram",
               eps: float = _ns.DEFAULT_EPS):
    """One Dion3 step on one matrix.  Returns a dict with the new momentum,
    the new weights (float64), the kept indices and the orthogonalized
    block O (k x n)."""
    mode = _momentum.ACCUM if ef_mode == EF_ROWS else _momentum.EMA
    B = _momentum.momentum_update(M, G, mu, mode)
    keys = _momentum.row_sqnorms(B)
    idx = select_rows(keys, rho)
    X0, factor = gather_normalize(B, idx, keys, eps)
    if variant == "gram":
        O = _ns.gram_newton_schulz(X0, iters, coeffs, safety, eps,
                                   normalize=False, restart_after=restart_after)
    else:
        O = _ns.newton_schulz(X0, iters, coeffs, safety, eps, normalize=False)
    M_new = ef_write(B, idx, mu) if ef_mode == EF_ROWS else B
    W_new = _apply.apply_update(W, O, idx, lr, scale, wd)
    return {"M": M_new, "W": W_new, "idx": idx, "O": O, "keys": keys,
            "factor": factor, "B": B}
