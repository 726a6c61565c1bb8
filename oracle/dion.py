"""Dion and Orth-Dion low-rank step (oracle).

Sources ("Orth-Dion: Eliminating Geometric Mismatch in Distributed Low-Rank
Spectral Optimization", gist.science):

* Problem Statement: Dion approximates Muon with rank-r factors
  (r << min(m, n)) obtained from a single power-iteration step per optimizer
  step.
* The Geometric Insight: Dion finishes the right factor with column
  normalization, which keeps the column span but not orthogonality, so the
  update's operator norm can reach sqrt(r).
* Orth-Dion: the same power iteration and residual buffer, with the column
  normalization replaced by QR orthogonalization of the right factor; the
  update becomes a partial isometry.
* Theoretical Contributions: an error-feedback coefficient beta (beta = 1 is
  Dion's buffer).

Step (one matrix; readings listed in the design notes):

    B      = M + G                         (fp32-stored buffer)
    P      = orth(B Q_prev)                (m x r, Householder QR, R diag > 0)
    R      = B^T P                         (n x r)
    Q_new  = ColNorm(R)   (Dion)   or   orth(R)   (Orth-Dion)
    M_new  = beta B - (beta - mu) P R^T    (beta = 1: B - (1 - mu) P R^T)
    O      = P Q_new^T
    W_new  = (1 - lr wd) W - lr scale O

ColNorm(R)_j = R_j / (||R_j||_2 + eps), eps = 1e-8.

Ada-Orth-Dion ("Ada-Orth-Dion": the working rank of each layer follows an
entropy-based estimate of its intrinsic dimensionality, derived from the
power-iteration factors; the pages do not define the estimator).  Reading:
sigma_j = ||R_j||_2, the power iteration's estimates of B's leading singular
values, and the estimate is the effective rank exp(H(p)),
p_j = sigma_j^2 / sum_k sigma_k^2, H the Shannon entropy.  Parity of this
estimator against the method is unpinned (the pages give no formula); the
function itself is pinned by its closed forms.

TEST INFRASTRUCTURE: see the package docstring.
"""
from __future__ import annotations

import numpy as np

from . import apply as _apply

COLNORM = 0
QR = 1
COLNORM_EPS = 1e-8


def householder_qr(A):
    """Thin QR of a tall matrix (m >= r) by Householder reflections.

    Returns (Q, R) with Q m x r having orthonormal columns, R r x r upper
    triangular, and the signs fixed so that diag(R) >= 0 (which makes the
    factorization unique for full column rank).
    """
    A = np.array(A, dtype=np.float64)
    m, r = A.shape
    if m < r:
        raise ValueError("householder_qr needs rows >= cols")
    Rw = A.copy()
    vs = []
    for j in range(r):
        x = Rw[j:, j]
        normx = np.sqrt(np.dot(x, x))
        if normx == 0.0:
            vs.append(None)
            continue
        v = x.copy()
        v[0] += normx if x[0] >= 0 else -normx
        vnorm2 = np.dot(v, v)
        # Rw[j:, j:] <- (I - 2 v v^T / v^T v) Rw[j:, j:]
        Rw[j:, j:] -= np.outer(v, (2.0 / vnorm2) * (v @ Rw[j:, j:]))
        vs.append((v, vnorm2))
    # Q = H_1 H_2 ... H_r applied to the first r columns of the identity.
    Q = np.zeros((m, r))
    Q[:r, :r] = np.eye(r)
    for j in range(r - 1, -1, -1):
        if vs[j] is None:
            continue
        v, vnorm2 = vs[j]
        Q[j:, :] -= np.outer(v, (2.0 / vnorm2) * (v @ Q[j:, :]))
    R = np.triu(Rw[:r, :r])
    signs = np.where(np.diag(R) < 0, -1.0, 1.0)
    return Q * signs[None, :], R * signs[:, None]


def orth(A):
    """Orthonormal basis of the columns of ``A`` (the Q of householder_qr)."""
    return householder_qr(A)[0]


def colnorm(R, eps: float = COLNORM_EPS):
    """Each column divided by (its 2-norm + eps)."""
    R = np.asarray(R, dtype=np.float64)
    norms = np.sqrt(np.sum(R * R, axis=0))
    return R / (norms + eps)[None, :]


def dion_step(M, G, Q_prev, W, mu: float, lr: float, scale: float,
              norm_mode: int = COLNORM, beta: float = 1.0, wd: float = 0.0,
              eps: float = COLNORM_EPS, state_dtype=np.float32):
    """One Dion (``COLNORM``) or Orth-Dion (``QR``) step on one matrix.

    ``Q_prev`` is n x r.  Returns a dict with the new buffer ``M`` (rounded
    to ``state_dtype``), ``Q`` (n x r, float64), ``W`` (float64) and the
    intermediates ``B``, ``P``, ``R``, ``O``.
    """
    M64 = np.asarray(M, dtype=np.float64)
    G64 = np.asarray(G, dtype=np.float64)
    B = M64 + G64
    if state_dtype is not None:
        B = B.astype(state_dtype).astype(np.float64)
    P = orth(B @ np.asarray(Q_prev, dtype=np.float64))
    R = B.T @ P
    if norm_mode == COLNORM:
        Q_new = colnorm(R, eps)
    elif norm_mode == QR:
        Q_new = orth(R)
    else:
        raise ValueError(f"unknown norm mode {norm_mode}")
    mu = float(np.float32(mu))
    beta = float(np.float32(beta))
    M_new = beta * B - (beta - mu) * (P @ R.T)
    if state_dtype is not None:
        M_new = M_new.astype(state_dtype)
    O = P @ Q_new.T
    W_new = _apply.apply_update(W, O, None, lr, scale, wd)
    return {"M": M_new, "Q": Q_new, "W": W_new, "B": B, "P": P, "R": R,
            "O": O, "sigma": np.linalg.norm(R, axis=0)}


def effective_rank(sigma) -> float:
    """exp(-sum_j p_j ln p_j), p_j = sigma_j^2 / sum_k sigma_k^2 (terms with
    p_j = 0 contribute 0); 0 when every sigma_j is 0."""
    s2 = np.asarray(sigma, dtype=np.float64) ** 2
    tot = s2.sum()
    if tot <= 0.0:
        return 0.0
    p = s2[s2 > 0] / tot
    return float(np.exp(-np.sum(p * np.log(p))))
