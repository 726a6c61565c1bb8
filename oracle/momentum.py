"""Momentum update (oracle, float64 arithmetic, fp32-stored state).

The Dion3 summary ("Dion3：全栈正交更新", 输入输出流程) orders a step as
"update momentum -> select rows -> Gram Newton-Schulz -> update weights".
Two forms are used:

* EMA (Muon form):           M <- mu * M + G
* ACCUM (error-feedback form): B = M + G, written over M; the orthogonalized
  part is removed from it afterwards (Dion's residual buffer, "Orth-Dion",
  Orth-Dion section; Dion3's error feedback, Dion3 summary 核心模块).

The momentum state is kept in fp32 (the workloads hold fp32 momentum), so the
oracle rounds the updated state to fp32 after computing it in float64.  The
row keys used by the row-selection rule are the float64 sums of squares of the
stored fp32 values.

TEST INFRASTRUCTURE: see the package docstring.
"""
from __future__ import annotations

import numpy as np

EMA = 0
ACCUM = 1


def momentum_update(M, G, mu: float, mode: int = EMA, state_dtype=np.float32):
    """Return the new momentum state (rounded to ``state_dtype``).

    ``M`` and ``G`` are arrays of the same shape; they are read as float64.
    ``mu`` is taken at fp32 precision (the value the kernels receive).
    """
    M64 = np.asarray(M, dtype=np.float64)
    G64 = np.asarray(G, dtype=np.float64)
    mu64 = float(np.float32(mu))
    if mode == EMA:
        new = mu64 * M64 + G64
    elif mode == ACCUM:
        new = M64 + G64
    else:
        raise ValueError(f"unknown momentum mode {mode}")
    if state_dtype is None:
        return new
    return new.astype(state_dtype)


def row_sqnorms(B) -> np.ndarray:
    """Float64 sum over each row of the squared entries of ``B``."""
    B64 = np.asarray(B, dtype=np.float64)
    return np.einsum("ij,ij->i", B64, B64)
