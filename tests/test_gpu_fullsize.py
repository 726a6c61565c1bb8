"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times, on outputs the oracle can compute one matrix at a time;
bit-exact determinism; the bounded-wait failure path."""
import ctypes
import math

import numpy as np
import pytest
import torch

import orthonormalized_update_optimizers_b200 as ouo
from orthonormalized_update_optimizers_b200 import _lib as L
from orthonormalized_update_optimizers_b200 import synth
from oracle import dion as odion
from oracle import dion3 as odion3
from oracle import ns as ons

from ._util import TOL_BF16, rel_fro, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
RHO, MU, LR = 0.125, 0.95, 0.02


def _dion3_step(Ms, Gs, Ws, scales, ef=True):
    keys = torch.empty(sum(M.shape[0] for M in Ms), dtype=torch.float64, device=DEV)
    ouo.dion_momentum_update(Ms, Gs, MU, "accum" if ef else "ema", keys)
    ks = [ouo.dion3_num_selected(M.shape[0], RHO) for M in Ms]
    idx = torch.empty(sum(ks), dtype=torch.int32, device=DEV)
    X0 = [torch.empty(k, M.shape[1], dtype=torch.bfloat16, device=DEV) for k, M in zip(ks, Ms)]
    sc = torch.empty(len(Ms), dtype=torch.float32, device=DEV)
    ouo.dion3_select_rows(Ms, keys, RHO, idx, X0, sc, ef=ef, mu=MU)
    O = [torch.empty_like(x) for x in X0]
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    ouo.gram_ns_orthogonalize(X0, O, ouo.ns_params(normalize=False), status=status)
    ouo.apply_update(Ws, O, LR, idx=idx, scale=scales)
    torch.cuda.synchronize()
    assert status.item() == 0
    return idx.cpu().numpy(), ks, O


def test_llama8b_shaped_step_sampled_against_oracle():
    # The benchmark's workload and batching (all 224 matrices in one step);
    # layers 0 and 31 of every projection checked against the oracle.
    shapes = synth.llama8b_shapes(32)
    Gs, Ms, Ws = [], [], []
    for i, (_, m, n) in enumerate(shapes):
        Gs.append(synth.lowrank_plus_noise(m, n, 32, 0.01, synth.seed_for(3, i),
                                           torch.bfloat16, DEV))
        Ms.append(torch.zeros(m, n, dtype=torch.float32, device=DEV))
        Ws.append(synth.gaussian((m, n), synth.seed_for(3, 1000 + i), 0.02,
                                 torch.bfloat16, DEV))
    scales = [math.sqrt(max(1.0, m / n)) for _, m, n in shapes]
    sample = list(range(7)) + list(range(31 * 7, 32 * 7))
    W0 = {i: to64(Ws[i]) for i in sample}
    G0 = {i: to64(Gs[i]) for i in sample}
    idx, ks, O = _dion3_step(Ms, Gs, Ws, scales)
    offs = np.concatenate([[0], np.cumsum(ks)])
    for i in sample:
        m, n = shapes[i][1], shapes[i][2]
        ref = odion3.dion3_step(np.zeros((m, n), np.float32), G0[i], W0[i], MU, RHO, LR,
                                scales[i])
        assert np.array_equal(idx[offs[i]:offs[i + 1]], ref["idx"]), shapes[i][0]
        assert rel_fro(to64(O[i]), ref["O"]) <= TOL_BF16, shapes[i][0]
        Mg = Ms[i].cpu().numpy()
        assert np.count_nonzero(Mg != ref["M"]) <= Mg.size // 100000 + 1
        # bf16 weights: rows outside S are untouched; on S the stored value
        # differs from the oracle's float64 one by at most one bf16 rounding
        # (<= 2^-9 relative, bounded here by 2^-8) plus the update's own
        # tolerance.  A missing, misplaced or sign-flipped update exceeds it.
        Wg = to64(Ws[i])
        S = ref["idx"]
        notS = np.setdiff1d(np.arange(m), S)
        assert np.array_equal(Wg[notS], W0[i][notS])
        upd = ref["W"][S] - W0[i][S]
        err = np.linalg.norm(Wg[S] - ref["W"][S])
        assert err <= 2.0 ** -8 * np.linalg.norm(ref["W"][S]) + TOL_BF16 * np.linalg.norm(upd)
        assert np.linalg.norm(upd) > 2.0 ** -8 * np.linalg.norm(ref["W"][S])  # the check has teeth
    del Gs, Ms, Ws, O
    torch.cuda.empty_cache()


def test_dion3_batch_16x1024x4096():
    shapes = [(1024, 4096)] * 16
    Gs = [synth.lowrank_plus_noise(m, n, 64, 0.02, synth.seed_for(1, i), torch.bfloat16, DEV)
          for i, (m, n) in enumerate(shapes)]
    Ms = [torch.zeros(s, dtype=torch.float32, device=DEV) for s in shapes]
    Ws = [torch.zeros(s, dtype=torch.float32, device=DEV) for s in shapes]
    G0 = [to64(g) for g in Gs]
    idx, ks, O = _dion3_step(Ms, Gs, Ws, [1.0] * 16)
    for i in range(16):
        ref = odion3.dion3_step(np.zeros(shapes[i], np.float32), G0[i],
                                np.zeros(shapes[i]), MU, RHO, LR, 1.0)
        assert np.array_equal(idx[128 * i:128 * (i + 1)], ref["idx"])
        assert rel_fro(to64(O[i]), ref["O"]) <= TOL_BF16
        assert rel_fro(to64(Ws[i]), ref["W"]) <= TOL_BF16


def test_gram_ns_full_16x1024x4096_sampled():
    Xs = [synth.lowrank_plus_noise(1024, 4096, 64, 0.02, synth.seed_for(1, i), torch.bfloat16, DEV)
          for i in range(16)]
    Os = [torch.empty_like(x) for x in Xs]
    ouo.gram_ns_orthogonalize(Xs, Os, ouo.ns_params())
    torch.cuda.synchronize()
    for i in (0, 7, 15):
        ref = ons.gram_newton_schulz(to64(Xs[i]), 5, restart_after=(3,))
        assert rel_fro(to64(Os[i]), ref) <= TOL_BF16


def _clone(ts):
    return [t.clone() for t in ts]


def test_steps_are_deterministic_across_a_state_snapshot():
    # 4 steps straight == 2 steps, snapshot (clone) of the state, 2 more steps:
    # bit-identical (fixed-order reductions, no floating-point atomics).
    shapes = [(512, 2048), (2048, 512), (256, 1024)]
    Gs = [[synth.lowrank_plus_noise(m, n, 32, 0.01, 500 + 10 * s + i, torch.bfloat16, DEV)
           for i, (m, n) in enumerate(shapes)] for s in range(4)]
    M1 = [torch.zeros(s, device=DEV) for s in shapes]
    W1 = [torch.zeros(s, dtype=torch.bfloat16, device=DEV) for s in shapes]
    for s in range(4):
        _dion3_step(M1, Gs[s], W1, [1.0, 2.0, 1.0])
    M2 = [torch.zeros(s, device=DEV) for s in shapes]
    W2 = [torch.zeros(s, dtype=torch.bfloat16, device=DEV) for s in shapes]
    for s in range(2):
        _dion3_step(M2, Gs[s], W2, [1.0, 2.0, 1.0])
    M3, W3 = _clone(M2), _clone(W2)
    del M2, W2
    for s in range(2, 4):
        _dion3_step(M3, Gs[s], W3, [1.0, 2.0, 1.0])
    for a, b in zip(M1 + W1, M3 + W3):
        assert torch.equal(a, b)
    # Dion: same property
    m, n, r = 512, 768, 64
    q0 = odion.orth(synth.dion_q0(n, r, 1).double().numpy()).astype(np.float32)
    p = ouo.dion_params(rank=r, norm_mode="qr")
    G = synth.lowrank_plus_noise(m, n, 64, 0.02, 9, torch.bfloat16, DEV)
    states = []
    for split in (False, True):
        M = torch.zeros(m, n, device=DEV)
        W = torch.zeros(m, n, device=DEV)
        Q = torch.tensor(q0.T.copy(), device=DEV)
        for s in range(4):
            if split and s == 2:
                M, W, Q = M.clone(), W.clone(), Q.clone()
            ouo.dion_lowrank_step([M], [G], [Q], [W], p)
        torch.cuda.synchronize()
        states.append((M, W, Q))
    for a, b in zip(*states):
        assert torch.equal(a, b)


def test_bounded_wait_reports_timeout_and_context_survives():
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    rc = L.lib().ouo_debug_wait_timeout(ctypes.c_void_p(status.data_ptr()),
                                        50_000_000, None)
    assert rc == 0
    torch.cuda.synchronize()
    assert status.item() == L.OUO_STATUS_TIMEOUT
    # the context is intact: a normal call still runs and reports nothing
    X = synth.gaussian((128, 512), 3, 1.0, torch.bfloat16, DEV)
    O = torch.empty_like(X)
    st2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    ouo.gram_ns_orthogonalize([X], [O], ouo.ns_params(), status=st2)
    torch.cuda.synchronize()
    assert st2.item() == 0
    assert rel_fro(to64(O), ons.gram_newton_schulz(to64(X), 5)) <= TOL_BF16


# Shape sweep (square to 16x wide, bf16 low-rank(64) + noise), standard and
# Gram NS with normalization on.  Sizes the oracle finishes in seconds are
# checked matrix by matrix; the largest shapes by the identity both iterations
# satisfy in exact arithmetic (Gram NS computes the standard iteration's
# polynomial), within twice the per-path tolerance.
SWEEP_ORACLE = [(512, 512), (512, 8192), (1024, 1024), (1024, 16384), (2048, 2048),
                (2048, 8192), (1024, 4096)]
SWEEP_LARGE = [(4096, 16384), (8192, 8192), (4096, 65536), (8192, 131072)]


@pytest.mark.parametrize("shape", SWEEP_ORACLE)
def test_shape_sweep_against_oracle(shape):
    m, n = shape
    nb = 3
    Xs = ouo.batch_empty([shape] * nb, torch.bfloat16, DEV)
    for i, x in enumerate(Xs):
        x.copy_(synth.lowrank_plus_noise(m, n, 64, 0.02, synth.seed_for(4, 100 * i + n // m),
                                         torch.bfloat16, DEV))
    Os = [torch.empty_like(x) for x in Xs]
    Og = [torch.empty_like(x) for x in Xs]
    ouo.ns_orthogonalize(Xs, Os, ouo.ns_params())
    ouo.gram_ns_orthogonalize(Xs, Og, ouo.ns_params())
    torch.cuda.synchronize()
    for i in (0, nb - 1):
        X64 = to64(Xs[i])
        assert rel_fro(to64(Os[i]), ons.newton_schulz(X64, 5)) <= TOL_BF16
        assert rel_fro(to64(Og[i]), ons.gram_newton_schulz(X64, 5, restart_after=(3,))) <= TOL_BF16


@pytest.mark.parametrize("shape", SWEEP_LARGE)
def test_shape_sweep_large_gram_equals_standard(shape):
    m, n = shape
    X = synth.lowrank_plus_noise(m, n, 64, 0.02, synth.seed_for(4, n // m), torch.bfloat16, DEV)
    Os, Og = torch.empty_like(X), torch.empty_like(X)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    ouo.ns_orthogonalize([X], [Os], ouo.ns_params(), status=status)
    ouo.gram_ns_orthogonalize([X], [Og], ouo.ns_params(), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    d = (Os.float() - Og.float()).norm() / Os.float().norm()
    assert torch.isfinite(Og.float()).all()
    assert d.item() <= 2 * TOL_BF16
    # the output is neither vanishing nor blown up: ||O||_F^2 / m is the mean
    # of the squared output singular values, each at most 1.2024^2 (the upper
    # edge of the quintic's band), and most of them are near one here
    ms = (Og.float().norm() ** 2 / m).item()
    assert 0.3 <= ms <= 1.2024 ** 2
    del X, Os, Og
    torch.cuda.empty_cache()


def test_chunked_step_equals_whole_step_bitwise():
    # A matrix's result does not depend on the batch it is stepped in: two
    # layers stepped as one batch, and as two one-layer chunks through views
    # of the same row-key / index / X0 / O buffers (the end-to-end schedule of
    # the benchmark), give bit-identical momentum, indices, O and weights.
    shapes = synth.llama8b_shapes(2)
    mn = [(m, n) for _, m, n in shapes]
    ks = [ouo.dion3_num_selected(m, RHO) for m, _ in mn]
    res = []
    for chunked in (False, True):
        G = [synth.lowrank_plus_noise(m, n, 32, 0.01, synth.seed_for(3, i), torch.bfloat16, DEV)
             for i, (m, n) in enumerate(mn)]
        M = [torch.zeros(m, n, device=DEV) for m, n in mn]
        W = [synth.gaussian((m, n), synth.seed_for(3, 1000 + i), 0.02, torch.bfloat16, DEV)
             for i, (m, n) in enumerate(mn)]
        keys = torch.empty(sum(m for m, _ in mn), dtype=torch.float64, device=DEV)
        idx = torch.empty(sum(ks), dtype=torch.int32, device=DEV)
        sc = torch.empty(len(mn), dtype=torch.float32, device=DEV)
        kn = [(k, n) for k, (_, n) in zip(ks, mn)]
        X0 = ouo.batch_empty(kn, torch.bfloat16, DEV)
        O = ouo.batch_empty(kn, torch.bfloat16, DEV)
        p = ouo.ns_params(normalize=False)
        spans = [(0, 7), (7, 14)] if chunked else [(0, 14)]
        kp = np.concatenate([[0], np.cumsum(ks)]).astype(int)
        rp = np.concatenate([[0], np.cumsum([m for m, _ in mn])]).astype(int)
        for a, b in spans:
            ouo.dion_momentum_update(M[a:b], G[a:b], MU, "accum", keys[rp[a]:rp[b]])
            ouo.dion3_select_rows(M[a:b], keys[rp[a]:rp[b]], RHO, idx[kp[a]:kp[b]], X0[a:b],
                                  sc[a:b], ef=True, mu=MU)
            ouo.gram_ns_orthogonalize(X0[a:b], O[a:b], p)
        ouo.apply_update(W, O, LR, idx=idx, scale=[1.0] * len(mn))
        torch.cuda.synchronize()
        res.append((M, W, idx.clone(), O))
    (M1, W1, i1, O1), (M2, W2, i2, O2) = res
    assert torch.equal(i1, i2)
    for a, b in zip(M1 + W1 + O1, M2 + W2 + O2):
        assert torch.equal(a, b)
