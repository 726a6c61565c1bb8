"""GPU parity of the Dion / Orth-Dion low-rank step (dion_lowrank_step)
against the oracle's dion_step: per step, the new buffer M, the new right
factor Q and the weight update, free-running from identical inputs."""
import numpy as np
import pytest
import torch

import orthonormalized_update_optimizers_b200 as ouo
from orthonormalized_update_optimizers_b200 import synth
from oracle import dion as odion

from ._util import TOL_BF16, rel_fro, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _q0(n, r, seed=1):
    # Dion's starting factor: a seeded N(0, 1) draw orthonormalized by the
    # oracle's QR, so both sides start from identical bytes.
    q = odion.orth(synth.dion_q0(n, r, seed).double().numpy())
    return q.astype(np.float32)


def _run(m, n, r, mode, steps, seed, w_dtype=torch.float32, beta=1.0,
         mu=0.95, lr=0.01, scale=1.0, g_same=True):
    G = synth.lowrank_plus_noise(m, n, min(64, m, n), 0.02, seed, torch.bfloat16, DEV)
    M = torch.zeros(m, n, dtype=torch.float32, device=DEV)
    W = synth.gaussian((m, n), seed + 7, 0.02, w_dtype, DEV)
    q0 = _q0(n, r)
    Qt = torch.tensor(q0.T.copy(), device=DEV)  # state is r x n (Q transposed)
    p = ouo.dion_params(rank=r, mu=mu, beta=beta, lr=lr,
                        norm_mode="qr" if mode == odion.QR else "colnorm")
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    Mr = np.zeros((m, n), dtype=np.float32)
    Wr = to64(W)
    Qr = q0.astype(np.float64)
    errs = []
    for step in range(steps):
        Gs = G if g_same else synth.lowrank_plus_noise(m, n, 64, 0.02, seed + 100 + step,
                                                       torch.bfloat16, DEV)
        W_before = to64(W)
        ouo.dion_lowrank_step([M], [Gs], [Qt], [W], p, scale=[scale], status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        ref = odion.dion_step(Mr, to64(Gs), Qr, Wr, mu, lr, scale, mode, beta=beta)
        e_m = rel_fro(to64(M), ref["M"])
        e_q = rel_fro(to64(Qt).T, ref["Q"])
        dW = to64(W) - W_before
        dW_ref = ref["W"] - Wr
        e_w = rel_fro(dW, dW_ref)
        errs.append((e_m, e_q, e_w))
        Mr, Wr, Qr = ref["M"], ref["W"], ref["Q"]
        if w_dtype == torch.bfloat16:
            Wr = to64(W)  # bf16 weights: compare the update, carry the stored value
    return errs


@pytest.mark.parametrize("mode", [odion.COLNORM, odion.QR])
@pytest.mark.parametrize("shape,r", [((256, 512), 32), ((300, 200), 16),
                                     ((512, 512), 128), ((96, 1000), 8)])
def test_dion_small(mode, shape, r):
    errs = _run(*shape, r, mode, steps=3, seed=sum(shape) + r)
    for e_m, e_q, e_w in errs:
        assert e_m <= TOL_BF16 and e_q <= TOL_BF16 and e_w <= TOL_BF16, errs


def test_dion_bf16_weights_and_beta():
    errs = _run(384, 640, 48, odion.QR, steps=2, seed=5, w_dtype=torch.bfloat16,
                beta=0.5, lr=0.05, scale=2.0)
    for e_m, e_q, e_w in errs:
        assert e_m <= TOL_BF16 and e_q <= TOL_BF16 and e_w <= 3e-2, errs


@pytest.mark.parametrize("mode", [odion.COLNORM, odion.QR])
def test_dion_4096_rank256_20_steps(mode):
    # one 4096 x 4096 bf16 low-rank(64) + noise gradient (the same each
    # step), r = 256, mu = 0.95, 20 steps free-running on both sides
    errs = _run(4096, 4096, 256, mode, steps=20, seed=2000)
    for step, (e_m, e_q, e_w) in enumerate(errs):
        assert e_m <= TOL_BF16 and e_q <= TOL_BF16 and e_w <= TOL_BF16, (step, errs)


@pytest.mark.parametrize("mode", [odion.COLNORM, odion.QR])
@pytest.mark.parametrize("shape,r,steps", [((1024, 768), 300, 3), ((1536, 1536), 512, 3)])
def test_dion_wide_ranks(mode, shape, r, steps):
    # ranks above 128 take the blocked multi-CTA Cholesky (r = 300 is not a
    # multiple of its 32-wide blocks)
    errs = _run(*shape, r, mode, steps=steps, seed=r)
    for e_m, e_q, e_w in errs:
        assert e_m <= TOL_BF16 and e_q <= TOL_BF16 and e_w <= TOL_BF16, errs


def test_orth_dion_rank_1024():
    errs = _run(2048, 2048, 1024, odion.QR, steps=2, seed=1024)
    for e_m, e_q, e_w in errs:
        assert e_m <= TOL_BF16 and e_q <= TOL_BF16 and e_w <= TOL_BF16, errs


def test_dion_orthonormal_factors_and_isometry():
    # Orth-Dion's update is a partial isometry: singular values of the
    # applied update P Q^T all equal one (nu_t = 1).
    m, n, r = 512, 768, 64
    G = synth.lowrank_plus_noise(m, n, 64, 0.02, 77, torch.bfloat16, DEV)
    M = torch.zeros(m, n, dtype=torch.float32, device=DEV)
    W = torch.zeros(m, n, dtype=torch.float32, device=DEV)
    Qt = torch.tensor(_q0(n, r).T.copy(), device=DEV)
    p = ouo.dion_params(rank=r, lr=1.0, norm_mode="qr")
    ouo.dion_lowrank_step([M], [G], [Qt], [W], p)
    torch.cuda.synchronize()
    q = to64(Qt)
    assert np.max(np.abs(q @ q.T - np.eye(r))) <= 1e-4
    sv = np.linalg.svd(-to64(W), compute_uv=False)
    assert np.max(np.abs(sv[:r] - 1.0)) <= 1e-3 and np.max(sv[r:]) <= 1e-3
