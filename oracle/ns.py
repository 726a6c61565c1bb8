"""Quintic Newton-Schulz and Gram Newton-Schulz (oracle).

Sources:

* "Dion3: Full-Stack Orthogonal Updates", Abstract: Muon's orthogonalization
  is a cubic-time Newton-Schulz step; Gram Newton-Schulz lowers its FLOP cost.
* "Dion3：全栈正交更新", 核心洞察 and 核心模块: Gram-NS works on the symmetric
  Gram matrix of the momentum instead of on the full matrix, and is kept
  stable by restarts and safety factors; 局限 names spurious negative
  eigenvalues and eigenvector drift as what the restarts repair.

Standard NS (one iteration, coefficients a, b, c):

    A = X X^T,   X <- a X + (b A + c A^2) X

so each singular value maps through p(x) = a x + b x^3 + c x^5.

Gram NS keeps X0 fixed and iterates on the k x k matrices only.  With
H_t = a I + b A + c A^2 the standard iterate is X_t = H_t X_{t-1}; hence
X_t = Q_t X0 with Q_t = H_t Q_{t-1} (Q_0 = I) and the next Gram matrix is
A_t = X_t X_t^T = H_t A_{t-1} H_t.  The accumulated polynomial Q is applied
to X0 once at the end.  A restart after iteration t materializes
X0 <- Q_t X0, recomputes A = X0 X0^T and resets Q = I.  In exact arithmetic
the result equals standard NS for any restart schedule.

Readings taken where the pages are silent (each listed in the design notes):

* Normalization X0 = X / (||X||_F + eps), eps = 1e-7, before the first
  iteration; ``normalize=False`` skips it for inputs already normalized.
* Orientation: a matrix with more rows than columns is transposed, processed,
  and transposed back (identical result in exact arithmetic).
* Safety factor s: every iteration uses p(x / s), i.e. coefficients
  (a / s, b / s^3, c / s^5); s = 1 leaves them unchanged.
* Quadratic term: H = a I + b A + c (A A).
* Restart position: a list of iteration numbers after which to restart
  (default: after iteration 3 of 5).

TEST INFRASTRUCTURE: see the package docstring.
"""
from __future__ import annotations

import numpy as np

# Muon's fixed quintic Newton-Schulz coefficients.
MUON_COEFFS = (3.4445, -4.7750, 2.0315)
DEFAULT_EPS = 1e-7


def scaled_coeffs(coeffs=MUON_COEFFS, safety=1):
    """Coefficients of p(x / s): (a / s, b / s^3, c / s^5)."""
    a, b, c = coeffs
    s = safety
    return (a / s, b / (s * s * s), c / (s * s * s * s * s))


def frobenius_normalize(X, eps: float = DEFAULT_EPS):
    """Return (X / (||X||_F + eps), the factor applied)."""
    X = np.asarray(X, dtype=np.float64)
    fro = float(np.sqrt(np.sum(X * X)))
    factor = 1.0 / (fro + eps)
    return X * factor, factor


def _identity_like(k, like):
    if like.dtype == object:
        eye = np.zeros((k, k), dtype=object)
        one = like.flat[0] * 0 + 1  # keeps the scalar type (e.g. Fraction)
        zero = like.flat[0] * 0
        eye[:, :] = zero
        for i in range(k):
            eye[i, i] = one
        return eye
    return np.eye(k, dtype=like.dtype)


def _prepare(X, normalize, eps):
    if X.dtype != object:
        X = np.asarray(X, dtype=np.float64)
    transposed = X.shape[0] > X.shape[1]
    if transposed:
        X = X.T.copy()
    if normalize:
        X, _ = frobenius_normalize(X, eps)
    return X, transposed


def newton_schulz(X, iters: int = 5, coeffs=MUON_COEFFS, safety=1,
                  eps: float = DEFAULT_EPS, normalize: bool = True):
    """Standard quintic Newton-Schulz: ``iters`` iterations of
    X <- a X + (b A + c A^2) X with A = X X^T."""
    X, transposed = _prepare(X, normalize, eps)
    a, b, c = scaled_coeffs(coeffs, safety)
    for _ in range(iters):
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    return X.T if transposed else X


def gram_newton_schulz(X, iters: int = 5, coeffs=MUON_COEFFS, safety=1,
                       eps: float = DEFAULT_EPS, normalize: bool = True,
                       restart_after=(3,)):
    """Gram Newton-Schulz with restarts (see the module docstring).

    ``restart_after`` lists iteration numbers t (1-based, t < iters) after
    which X0 <- Q X0, A <- X0 X0^T, Q <- I.
    """
    X0, transposed = _prepare(X, normalize, eps)
    a, b, c = scaled_coeffs(coeffs, safety)
    restarts = {int(t) for t in restart_after if 0 < int(t) < iters}
    k = X0.shape[0]
    A = X0 @ X0.T
    Q = _identity_like(k, A)
    for t in range(1, iters + 1):
        eye = _identity_like(k, A)
        H = a * eye + b * A + c * (A @ A)
        Q = H @ Q
        if t == iters:
            break
        if t in restarts:
            X0 = Q @ X0
            A = X0 @ X0.T
            Q = _identity_like(k, A)
        else:
            A = H @ (H @ A)
    out = Q @ X0
    return out.T if transposed else out
