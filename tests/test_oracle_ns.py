"""Pins for the oracle's Newton-Schulz and Gram Newton-Schulz.

Each test fixes the oracle to something other than itself: exact rational
arithmetic, the SVD (spectral mapping of the odd polynomial), the textbook
cubic Newton-Schulz limit (the polar factor), invariances of the iteration.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import ns

A_, B_, C_ = ns.MUON_COEFFS


def _rng(seed):
    return np.random.default_rng(seed)


def _poly_iterate(x, iters, coeffs, safety=1.0):
    # scalar image of the singular values: p(x/s) with p(x) = a x + b x^3 + c x^5
    a, b, c = coeffs
    for _ in range(iters):
        y = x / safety
        x = a * y + b * y ** 3 + c * y ** 5
    return x


@pytest.mark.parametrize("shape", [(64, 256), (256, 64), (48, 48)])
@pytest.mark.parametrize("restarts", [(), (1,), (3,), (2, 4)])
@pytest.mark.parametrize("safety", [1.0, 1.01])
def test_gram_equals_standard_fp64(shape, restarts, safety):
    X = _rng(1).standard_normal(shape)
    a = ns.newton_schulz(X, 5, safety=safety)
    b = ns.gram_newton_schulz(X, 5, safety=safety, restart_after=restarts)
    assert np.max(np.abs(a - b)) <= 1e-10


def _exact_coeffs():
    return (Fraction("3.4445"), Fraction("-4.7750"), Fraction("2.0315"))


@pytest.mark.parametrize("restarts", [(), (1,), (2,)])
def test_gram_equals_standard_exact_rational(restarts):
    # 8 x 16 matrix with entries in {-2..2}/8, exact Fraction arithmetic:
    # Gram NS must reproduce standard NS bit for bit (no rounding anywhere).
    rng = _rng(7)
    ints = rng.integers(-2, 3, size=(8, 16))
    X = np.empty((8, 16), dtype=object)
    for i in range(8):
        for j in range(16):
            X[i, j] = Fraction(int(ints[i, j]), 8)
    coeffs = _exact_coeffs()
    a = ns.newton_schulz(X, 3, coeffs=coeffs, normalize=False)
    b = ns.gram_newton_schulz(X, 3, coeffs=coeffs, normalize=False,
                              restart_after=restarts)
    assert a.shape == b.shape == (8, 16)
    for i in range(8):
        for j in range(16):
            assert a[i, j] == b[i, j]


@pytest.mark.parametrize("shape", [(32, 80), (80, 32)])
@pytest.mark.parametrize("safety", [1.0, 1.01])
def test_closed_form_through_svd(shape, safety):
    # NS output = U p^5(sigma / ||X||_F) V^T because X X^T X = U S^3 V^T.
    X = _rng(2).standard_normal(shape)
    U, s, Vt = np.linalg.svd(X, full_matrices=False)
    shat = s / (np.linalg.norm(X) + ns.DEFAULT_EPS)
    expect = (U * _poly_iterate(shat, 5, ns.MUON_COEFFS, safety)) @ Vt
    for fn in (ns.newton_schulz, ns.gram_newton_schulz):
        out = fn(X, 5, safety=safety)
        assert np.max(np.abs(out - expect)) <= 1e-12


def test_textbook_cubic_converges_to_polar_factor():
    # With (a, b, c) = (3/2, -1/2, 0) the iteration is the textbook
    # Newton-Schulz for the orthogonal polar factor U V^T.
    X = _rng(3).standard_normal((24, 40))
    U, _, Vt = np.linalg.svd(X, full_matrices=False)
    polar = U @ Vt
    for fn in (ns.newton_schulz, ns.gram_newton_schulz):
        out = fn(X, 60, coeffs=(1.5, -0.5, 0.0))
        assert np.max(np.abs(out - polar)) <= 1e-10


def test_singular_value_band_and_vectors():
    # Muon's quintic p maps [0.01, 1] after 5 iterations into
    # [0.6818, 1.1344] (a scan of the scalar map; p's maximum on [0, 1] is
    # 1.2024 near x = 0.5545, a bound for any input).  The output keeps
    # the input's singular vectors: U^T O V is diagonal and positive.
    rng = _rng(4)
    U0 = np.linalg.qr(rng.standard_normal((64, 64)))[0]
    V0 = np.linalg.qr(rng.standard_normal((256, 64)))[0]
    s = np.geomspace(1.0, 0.1, 64)
    X = (U0 * s) @ V0.T
    out = ns.gram_newton_schulz(X, 5)
    sv = np.linalg.svd(out, compute_uv=False)
    shat_min = s.min() / np.linalg.norm(X)
    assert shat_min >= 0.01
    assert sv.max() <= 1.1344 and sv.min() >= 0.6818
    D = U0.T @ out @ V0
    assert np.max(np.abs(D - np.diag(np.diag(D)))) <= 1e-12
    assert np.all(np.diag(D) > 0)


def test_permutation_and_transpose_equivariance():
    rng = _rng(5)
    X = rng.standard_normal((40, 96))
    perm = rng.permutation(40)
    for fn in (ns.newton_schulz, ns.gram_newton_schulz):
        base = fn(X, 5)
        assert np.max(np.abs(fn(X[perm], 5) - base[perm])) <= 1e-12
        assert np.max(np.abs(fn(X.T, 5) - base.T)) <= 1e-12


def test_normalization_and_scale_invariance():
    X = _rng(6).standard_normal((16, 64))
    Xn, factor = ns.frobenius_normalize(X)
    assert abs(np.linalg.norm(Xn) - 1.0) <= 1e-6
    assert factor == pytest.approx(1.0 / (np.linalg.norm(X) + 1e-7))
    # the normalized iteration does not depend on the input's overall scale
    a = ns.gram_newton_schulz(X * 1e3, 5, eps=0.0)
    b0 = ns.gram_newton_schulz(X, 5, eps=0.0)
    assert np.max(np.abs(a - b0)) <= 1e-12
    b = ns.gram_newton_schulz(X, 5)
    # normalize=False on the normalized input equals normalize=True
    c = ns.gram_newton_schulz(Xn, 5, normalize=False)
    assert np.max(np.abs(c - b)) <= 1e-12


def test_safety_factor_is_input_rescaling():
    # p(x / s): the safety factor equals running the s = 1 iteration on X / s
    # for the first step only when iters = 1.
    X = _rng(8).standard_normal((12, 30))
    Xn, _ = ns.frobenius_normalize(X)
    a = ns.newton_schulz(Xn, 1, safety=1.05, normalize=False)
    b = ns.newton_schulz(Xn / 1.05, 1, safety=1.0, normalize=False)
    assert np.max(np.abs(a - b)) <= 1e-14


def test_zero_iterations_and_single_row():
    X = _rng(9).standard_normal((1, 50))
    out = ns.gram_newton_schulz(X, 5)
    # one row: p^5 of sigma_hat ~ 1 lands near the fixed point region
    expect = X / np.linalg.norm(X) * _poly_iterate(
        np.linalg.norm(X) / (np.linalg.norm(X) + 1e-7), 5, ns.MUON_COEFFS)
    assert np.max(np.abs(out - expect)) <= 1e-12
    out0 = ns.gram_newton_schulz(X, 0)
    assert np.max(np.abs(out0 - X / (np.linalg.norm(X) + 1e-7))) <= 1e-15
