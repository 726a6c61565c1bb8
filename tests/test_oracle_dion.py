"""Pins for the oracle's Householder QR, column normalization and the
Dion / Orth-Dion step: uniqueness of the positive-diagonal QR (matches the
LAPACK routine after sign fixing), the nu_t bounds the Orth-Dion page states,
error-feedback conservation, and full-rank recovery of the polar factor."""
import numpy as np
import pytest

from oracle import dion


def _rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("shape", [(300, 40), (64, 64), (4096, 8), (9, 1)])
def test_householder_qr(shape):
    A = _rng(0).standard_normal(shape)
    Q, R = dion.householder_qr(A)
    r = shape[1]
    assert Q.shape == shape and R.shape == (r, r)
    assert np.max(np.abs(Q.T @ Q - np.eye(r))) <= 1e-12
    assert np.max(np.abs(Q @ R - A)) <= 1e-12 * max(1.0, np.abs(A).max()) * 10
    assert np.array_equal(R, np.triu(R))
    assert np.all(np.diag(R) > 0)
    # unique with diag(R) > 0: equals LAPACK's QR after the same sign fix
    Ql, Rl = np.linalg.qr(A)
    sg = np.sign(np.diag(Rl))
    assert np.max(np.abs(Ql * sg - Q)) <= 1e-10


def test_colnorm_unit_columns():
    R = _rng(1).standard_normal((200, 16)) * np.arange(1, 17)
    Qc = dion.colnorm(R)
    norms = np.linalg.norm(Qc, axis=0)
    assert np.max(np.abs(norms - 1.0)) <= 1e-9  # eps = 1e-8 relative to norms >= ~10
    R2 = R / np.linalg.norm(R, axis=0)
    assert np.max(np.abs(dion.colnorm(R2, eps=0.0) - R2)) <= 1e-15
    # a zero column stays zero (no division by zero)
    R3 = R.copy()
    R3[:, 3] = 0
    assert np.all(dion.colnorm(R3)[:, 3] == 0)


def _step_inputs(m, n, r, seed):
    rng = _rng(seed)
    G = rng.standard_normal((m, n)).astype(np.float32)
    M = (0.1 * rng.standard_normal((m, n))).astype(np.float32)
    Q0 = dion.orth(rng.standard_normal((n, r)))
    W = rng.standard_normal((m, n)).astype(np.float32)
    return M, G, Q0, W


def test_nu_t_bounds():
    # The Geometric Insight: Dion's update P ColNorm(R)^T has operator norm in
    # [1, sqrt(r)];  Orth-Dion's update is a partial isometry (all nonzero
    # singular values equal to 1, nu_t = 1).
    r = 16
    M, G, Q0, W = _step_inputs(64, 96, r, 2)
    d = dion.dion_step(M, G, Q0, W, 0.95, 0.01, 1.0, dion.COLNORM)
    sv = np.linalg.svd(d["O"], compute_uv=False)
    assert 1.0 - 1e-9 <= sv.max() <= np.sqrt(r) + 1e-9
    o = dion.dion_step(M, G, Q0, W, 0.95, 0.01, 1.0, dion.QR)
    sv = np.linalg.svd(o["O"], compute_uv=False)
    assert np.max(np.abs(sv[:r] - 1.0)) <= 1e-12
    assert np.max(np.abs(sv[r:])) <= 1e-12


@pytest.mark.parametrize("mode", [dion.COLNORM, dion.QR])
def test_error_feedback_conservation(mode):
    M, G, Q0, W = _step_inputs(48, 40, 6, 3)
    d = dion.dion_step(M, G, Q0, W, 0.9, 0.05, 2.0, mode, state_dtype=None)
    B, P, R = d["B"], d["P"], d["R"]
    assert np.max(np.abs(d["M"] + (1 - float(np.float32(0.9))) * P @ R.T - B)) <= 1e-12
    assert np.max(np.abs(P.T @ P - np.eye(6))) <= 1e-12
    assert np.max(np.abs(R - B.T @ P)) <= 1e-12
    lr = float(np.float32(0.05))
    assert np.max(np.abs(d["W"] - (W - lr * 2.0 * P @ d["Q"].T))) <= 1e-12


def test_beta_reading_reduces_to_dion_at_one():
    M, G, Q0, W = _step_inputs(20, 30, 4, 4)
    a = dion.dion_step(M, G, Q0, W, 0.9, 0.1, 1.0, dion.QR, beta=1.0, state_dtype=None)
    b = dion.dion_step(M, G, Q0, W, 0.9, 0.1, 1.0, dion.QR, beta=0.1, state_dtype=None)
    B, P, R = b["B"], b["P"], b["R"]
    beta = float(np.float32(0.1))
    mu = float(np.float32(0.9))
    assert np.max(np.abs(b["M"] - (beta * (B - P @ R.T) + mu * P @ R.T))) <= 1e-12
    assert np.max(np.abs(a["M"] - (B - (1 - mu) * P @ R.T))) <= 1e-12


@pytest.mark.parametrize("mode", [dion.COLNORM, dion.QR])
def test_full_rank_power_iteration_recovers_polar_factor(mode):
    # m x n = 8 x 16, r = 8 = min(m, n), fixed B (momentum kept at zero so
    # error feedback is off), warm-started power iteration: P -> U, and the
    # update P Q^T -> U V^T (distinct singular values, positive-diagonal QR).
    rng = _rng(5)
    U = np.linalg.qr(rng.standard_normal((8, 8)))[0]
    V = np.linalg.qr(rng.standard_normal((16, 8)))[0]
    s = np.array([4.0, 3.2, 2.6, 2.0, 1.5, 1.1, 0.8, 0.5])
    Bm = (U * s) @ V.T
    Q = dion.orth(rng.standard_normal((16, 8)))
    Z = np.zeros((8, 16))
    for _ in range(200):
        # eps = 0: ColNorm's 1e-8 guard would bias the columns by 1e-8 / sigma
        d = dion.dion_step(Z, Bm, Q, Z, 0.95, 1.0, 1.0, mode, eps=0.0,
                           state_dtype=None)
        Q = d["Q"]
    assert np.max(np.abs(d["O"] - U @ V.T)) <= 1e-10


def test_single_step_shapes_and_dtypes():
    M, G, Q0, W = _step_inputs(33, 70, 5, 6)
    d = dion.dion_step(M, G, Q0, W, 0.95, 0.01, 1.0, dion.COLNORM)
    assert d["M"].dtype == np.float32 and d["M"].shape == (33, 70)
    assert d["Q"].shape == (70, 5) and d["P"].shape == (33, 5)
    assert np.max(np.abs(np.linalg.norm(d["Q"], axis=0) - 1)) <= 1e-7


# ---- Ada-Orth-Dion's effective-rank estimate (closed forms)
def test_effective_rank_closed_forms():
    assert dion.effective_rank(np.ones(37)) == pytest.approx(37.0, rel=1e-12)
    assert dion.effective_rank(np.array([0.0, 3.0, 0.0])) == pytest.approx(1.0, abs=1e-12)
    assert dion.effective_rank(np.array([2.0, 2.0, 0.0, 0.0])) == pytest.approx(2.0, rel=1e-12)
    assert dion.effective_rank(np.zeros(5)) == 0.0
    # energy split 3/4, 1/4: exp(-(3/4 ln 3/4 + 1/4 ln 1/4)) = 4 / 3^(3/4)
    assert dion.effective_rank(np.array([np.sqrt(3.0), 1.0])) == pytest.approx(
        4.0 / 3.0 ** 0.75, rel=1e-12)
    # scale and order invariance, and 1 <= erank <= r
    s = np.random.default_rng(4).random(50)
    e = dion.effective_rank(s)
    assert dion.effective_rank(7.5 * s[::-1]) == pytest.approx(e, rel=1e-12)
    assert 1.0 <= e <= 50.0


def test_effective_rank_of_a_dion_step_tracks_the_spectrum():
    # B = U diag(s) V^T with s = (1, ..., 1, 0, ...): a full-rank warm start
    # captures the spectrum, so the estimate equals the number of ones.
    rng = np.random.default_rng(6)
    m, n, r, k = 64, 48, 16, 6
    U = np.linalg.qr(rng.standard_normal((m, m)))[0][:, :n]
    V = np.linalg.qr(rng.standard_normal((n, n)))[0]
    s = np.zeros(n)
    s[:k] = 1.0
    B = (U * s) @ V.T
    Q0 = dion.orth(np.hstack([V[:, :k], rng.standard_normal((n, r - k))]))
    out = dion.dion_step(np.zeros((m, n)), B, Q0, np.zeros((m, n)), 0.95, 0.1, 1.0,
                          dion.QR, state_dtype=None)
    assert dion.effective_rank(out["sigma"]) == pytest.approx(float(k), rel=1e-9)
