"""Pins for the oracle's momentum update, Dion3 row selection, error feedback
and weight update: closed forms, brute-force sorting and conservation laws."""
import math

import numpy as np
import pytest

from oracle import apply, dion3, momentum, ns


def _rng(seed):
    return np.random.default_rng(seed)


def test_ema_closed_form_three_steps():
    # Three EMA steps from zero with the same G: M = (1 + mu + mu^2) G.
    G = _rng(0).standard_normal((8, 16)).astype(np.float32)
    M = np.zeros_like(G)
    for _ in range(3):
        M = momentum.momentum_update(M, G, 0.95, momentum.EMA)
    mu = float(np.float32(0.95))
    expect = (1 + mu + mu * mu) * G.astype(np.float64)
    assert M.dtype == np.float32
    assert np.max(np.abs(M - expect) / np.abs(expect)) <= 3e-7
    assert (1 + 0.95 + 0.95 ** 2) == pytest.approx(2.8525)


def test_accum_and_row_keys():
    rng = _rng(1)
    M = rng.standard_normal((5, 7)).astype(np.float32)
    G = rng.standard_normal((5, 7)).astype(np.float32)
    B = momentum.momentum_update(M, G, 0.5, momentum.ACCUM)
    assert np.array_equal(B, (M.astype(np.float64) + G).astype(np.float32))
    keys = momentum.row_sqnorms(B)
    for i in range(5):
        assert keys[i] == pytest.approx(sum(float(v) ** 2 for v in B[i]), rel=1e-15)


def _brute_topk(keys, k):
    order = sorted(range(len(keys)), key=lambda i: (-keys[i], i))
    return sorted(order[:k])


@pytest.mark.parametrize("m,rho", [(1, 0.125), (7, 0.125), (64, 0.125),
                                   (100, 0.3), (33, 1.0), (1000, 0.001)])
def test_select_rows_brute_force(m, rho):
    keys = _rng(m).random(m)
    idx = dion3.select_rows(keys, rho)
    k = max(1, min(m, math.ceil(rho * m - 1e-9)))
    assert len(idx) == k
    assert list(idx) == _brute_topk(list(keys), k)
    assert idx.dtype == np.int32


def test_select_rows_exact_ties():
    # duplicated rows, zero rows and integer rows: equal keys go to the lower
    # index, the output is ascending.
    rng = _rng(2)
    base = rng.integers(-3, 4, size=(6, 10)).astype(np.float32)
    B = np.concatenate([base, base[::-1], np.zeros((4, 10), np.float32),
                        base[:2]], axis=0)
    keys = momentum.row_sqnorms(B)
    for rho in (0.125, 0.25, 0.5, 0.75):
        idx = dion3.select_rows(keys, rho)
        assert list(idx) == _brute_topk(list(keys), len(idx))
    # all-equal keys: the first k rows
    assert list(dion3.select_rows(np.ones(16), 0.25)) == [0, 1, 2, 3]
    # all-zero rows
    assert list(dion3.select_rows(np.zeros(9), 0.125)) == [0, 1]


def test_num_selected_edges():
    assert dion3.num_selected(1024, 1 / 8) == 128
    assert dion3.num_selected(14336, 1 / 8) == 1792
    assert dion3.num_selected(1000, 1 / 8) == 125
    assert dion3.num_selected(1001, 1 / 8) == 126
    assert dion3.num_selected(5, 1e-6) == 1
    assert dion3.num_selected(5, 1.0) == 5


def test_gather_normalize_unit_frobenius():
    B = _rng(3).standard_normal((50, 40)).astype(np.float32)
    keys = momentum.row_sqnorms(B)
    idx = dion3.select_rows(keys, 0.2)
    X0, factor = dion3.gather_normalize(B, idx, keys)
    assert X0.shape == (10, 40)
    assert np.linalg.norm(X0) == pytest.approx(1.0, abs=1e-6)
    assert np.array_equal(X0 / factor, B[idx].astype(np.float64) * 1.0) or \
        np.max(np.abs(X0 / factor - B[idx])) <= 1e-12


def test_error_feedback_conservation():
    # kept rows: M_new + (1 - mu) B = B ; other rows: M_new = B.
    rng = _rng(4)
    M = rng.standard_normal((32, 24)).astype(np.float32)
    G = rng.standard_normal((32, 24)).astype(np.float32)
    W = rng.standard_normal((32, 24)).astype(np.float32)
    out = dion3.dion3_step(M, G, W, mu=0.95, rho=0.25, lr=0.01, scale=1.0)
    B = out["B"].astype(np.float64)
    S = out["idx"]
    notS = np.setdiff1d(np.arange(32), S)
    mu = float(np.float32(0.95))
    Mn = out["M"].astype(np.float64)
    assert np.max(np.abs(Mn[S] + (1 - mu) * B[S] - B[S])) <= 1e-6
    assert np.array_equal(out["M"][notS], out["B"][notS])
    # the weights move only on kept rows, by -lr * scale * O
    Wn = out["W"]
    assert np.array_equal(Wn[notS], W[notS].astype(np.float64))
    assert np.max(np.abs(Wn[S] - (W[S] - float(np.float32(0.01)) * out["O"]))) <= 1e-12
    # O is Gram NS of the normalized kept rows
    X0, _ = dion3.gather_normalize(B, S, momentum.row_sqnorms(out["B"]))
    O_std = ns.newton_schulz(X0, 5, normalize=False)
    assert np.max(np.abs(out["O"] - O_std)) <= 1e-10


def test_no_error_feedback_is_plain_ema():
    rng = _rng(5)
    M = rng.standard_normal((16, 8)).astype(np.float32)
    G = rng.standard_normal((16, 8)).astype(np.float32)
    W = np.zeros((16, 8), np.float32)
    out = dion3.dion3_step(M, G, W, 0.9, 0.25, 0.1, 1.0, ef_mode=dion3.EF_NONE)
    assert np.array_equal(out["M"], momentum.momentum_update(M, G, 0.9, momentum.EMA))


def test_permutation_of_kept_rows_commutes():
    # NS(P X) = P NS(X): the row order of the gather cannot matter.
    B = _rng(6).standard_normal((40, 30))
    keys = momentum.row_sqnorms(B)
    idx = dion3.select_rows(keys, 0.25)
    X0, _ = dion3.gather_normalize(B, idx, keys)
    perm = _rng(7).permutation(len(idx))
    a = ns.gram_newton_schulz(X0[perm], 5, normalize=False)
    b = ns.gram_newton_schulz(X0, 5, normalize=False)[perm]
    assert np.max(np.abs(a - b)) <= 1e-12


def test_apply_update_weight_decay():
    rng = _rng(8)
    W = rng.standard_normal((6, 5))
    O = rng.standard_normal((6, 5))
    out = apply.apply_update(W, O, None, lr=0.5, scale=2.0, wd=0.1)
    assert np.max(np.abs(out - ((1 - 0.05) * W - 1.0 * O))) <= 1e-7
    rows = np.array([1, 4])
    out2 = apply.apply_update(W, O[rows], rows, lr=0.5, scale=2.0)
    assert np.array_equal(out2[[0, 2, 3, 5]], W[[0, 2, 3, 5]])
    assert np.max(np.abs(out2[rows] - (W[rows] - O[rows]))) <= 1e-15
