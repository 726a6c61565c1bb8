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
         mu=0.95, lr=0.01, scale=1.0, g_same=True, wd=0.0, g_dtype=torch.bfloat16):
    G = synth.lowrank_plus_noise(m, n, min(64, m, n), 0.02, seed, g_dtype, DEV)
    M = torch.zeros(m, n, dtype=torch.float32, device=DEV)
    W = synth.gaussian((m, n), seed + 7, 0.02, w_dtype, DEV)
    q0 = _q0(n, r)
    Qt = torch.tensor(q0.T.copy(), device=DEV)  # state is r x n (Q transposed)
    p = ouo.dion_params(rank=r, mu=mu, beta=beta, lr=lr, wd=wd,
                        norm_mode="qr" if mode == odion.QR else "colnorm")
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    Mr = np.zeros((m, n), dtype=np.float32)
    Wr = to64(W)
    Qr = q0.astype(np.float64)
    errs = []
    for step in range(steps):
        Gs = G if g_same else synth.lowrank_plus_noise(m, n, 64, 0.02, seed + 100 + step,
                                                       g_dtype, DEV)
        W_before = to64(W)
        ouo.dion_lowrank_step([M], [Gs], [Qt], [W], p, scale=[scale], status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        ref = odion.dion_step(Mr, to64(Gs), Qr, Wr, mu, lr, scale, mode, beta=beta, wd=wd)
        e_m = rel_fro(to64(M), ref["M"])
        e_q = rel_fro(to64(Qt).T, ref["Q"])
        W_after = to64(W)
        dW = W_after - W_before
        dW_ref = ref["W"] - Wr
        if w_dtype == torch.bfloat16:
            # The kernel adds the update to the bf16 weights in fp32 and
            # stores the sum rounded to bf16: the stored dW carries one bf16
            # rounding of the weights (at most 2^-8 relative per element) on
            # top of the update's own error.  The error is stated as a
            # fraction of ||dW_ref|| after taking that rounding off.
            rnd = 2.0 ** -8 * np.linalg.norm(W_after)
            assert np.linalg.norm(dW_ref) > 4 * rnd  # the check has teeth
            e_w = max(0.0, np.linalg.norm(dW - dW_ref) - rnd) / np.linalg.norm(dW_ref)
        else:
            e_w = rel_fro(dW, dW_ref)
        errs.append((e_m, e_q, e_w))
        # the oracle carries its own state (it never takes a GPU value); with
        # bf16 weights the comparison is of the update dW, which does not
        # depend on the weights it is added to
        Mr, Wr, Qr = ref["M"], ref["W"], ref["Q"]
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
        assert e_m <= TOL_BF16 and e_q <= TOL_BF16 and e_w <= TOL_BF16, errs


@pytest.mark.parametrize("mode", [odion.COLNORM, odion.QR])
def test_dion_weight_decay(mode):
    # W <- (1 - lr wd) W - lr s P Q_new^T: the decoupled decay rides in the
    # in-place update's C0 coefficient
    errs = _run(512, 768, 64, mode, steps=2, seed=31, lr=0.05, wd=0.1, scale=1.5)
    for e_m, e_q, e_w in errs:
        assert e_m <= TOL_BF16 and e_q <= TOL_BF16 and e_w <= TOL_BF16, errs


def test_dion_fp32_gradient():
    # fp32 gradients take the momentum kernel's fp32 path; the rest of the
    # step is the same
    errs = _run(384, 512, 32, odion.QR, steps=2, seed=41, g_dtype=torch.float32)
    for e_m, e_q, e_w in errs:
        assert e_m <= TOL_BF16 and e_q <= TOL_BF16 and e_w <= TOL_BF16, errs


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
    # ranks above 224 take the cooperative multi-CTA Cholesky (r = 300 is
    # not a multiple of its 32-wide blocks)
    errs = _run(*shape, r, mode, steps=steps, seed=r)
    for e_m, e_q, e_w in errs:
        assert e_m <= TOL_BF16 and e_q <= TOL_BF16 and e_w <= TOL_BF16, errs


@pytest.mark.parametrize("mode", [odion.COLNORM, odion.QR])
@pytest.mark.parametrize("shape,r", [((256, 512), 8), ((300, 200), 40), ((640, 512), 65),
                                     ((512, 300), 100), ((768, 1024), 200),
                                     ((1024, 1024), 256)])
def test_one_cta_cholesky_ranks_up_to_256(mode, shape, r):
    # ranks up to 256 take the one-CTA blocked Cholesky: one block (r = 8),
    # ragged last blocks (40, 65, 100, 200) and all eight blocks (256)
    errs = _run(*shape, r, mode, steps=3, seed=3 * r + 1)
    for e_m, e_q, e_w in errs:
        assert e_m <= TOL_BF16 and e_q <= TOL_BF16 and e_w <= TOL_BF16, errs


@pytest.mark.parametrize("r", [96, 300])
def test_zero_gradient_takes_the_shifted_retry(r):
    # B = 0 makes every Gram matrix zero: the first factorization meets a
    # zero pivot, the shifted retry (tr S = 0, so the smallest positive
    # shift) succeeds, and the step leaves M at zero and W unchanged.  r = 96
    # runs the one-CTA Cholesky, r = 300 the cooperative one.
    m, n = 512, 384
    M = torch.zeros(m, n, device=DEV)
    G = torch.zeros(m, n, dtype=torch.bfloat16, device=DEV)
    W = synth.gaussian((m, n), 5, 0.02, torch.float32, DEV)
    W0 = W.clone()
    Qt = torch.tensor(_q0(n, r).T.copy(), device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    p = ouo.dion_params(rank=r, norm_mode="qr", lr=0.1)
    for _ in range(2):
        ouo.dion_lowrank_step([M], [G], [Qt], [W], p, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.count_nonzero(M).item() == 0
    assert torch.equal(W, W0)
    assert torch.isfinite(Qt).all()


def test_orth_dion_rank_1024():
    errs = _run(2048, 2048, 1024, odion.QR, steps=2, seed=1024)
    for e_m, e_q, e_w in errs:
        assert e_m <= TOL_BF16 and e_q <= TOL_BF16 and e_w <= TOL_BF16, errs


@pytest.mark.parametrize("r", [64, 256])
def test_cholesky_qr2_reaches_fp32_orthonormality(r):
    # The CholeskyQR2 of the right factor runs its Gram matrices and solves
    # as split-tf32 tensor-core products; plain tf32 would leave
    # ||Q Q^T - I|| near 1e-3, fp32-level products near 1e-6.
    m, n = 1024, 2048
    G = synth.lowrank_plus_noise(m, n, 32, 0.02, 91 + r, torch.bfloat16, DEV)
    M = torch.zeros(m, n, dtype=torch.float32, device=DEV)
    W = torch.zeros(m, n, dtype=torch.float32, device=DEV)
    Qt = torch.tensor(_q0(n, r).T.copy(), device=DEV)
    p = ouo.dion_params(rank=r, lr=1.0, norm_mode="qr")
    for _ in range(2):
        ouo.dion_lowrank_step([M], [G], [Qt], [W], p)
    torch.cuda.synchronize()
    q = to64(Qt)
    assert np.max(np.abs(q @ q.T - np.eye(r))) <= 1e-5


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


# ---- per-matrix working ranks (Ada-Orth-Dion) ----------------------------
def _state(shapes, ranks, seed=0):
    G = [synth.lowrank_plus_noise(m, n, min(64, m, n), 0.02, seed + i, torch.bfloat16, DEV)
         for i, (m, n) in enumerate(shapes)]
    W = [synth.gaussian((m, n), seed + 50 + i, 0.02, torch.float32, DEV)
         for i, (m, n) in enumerate(shapes)]
    Q = [torch.tensor(_q0(n, r, seed + 100 + i).T.copy(), device=DEV)
         for i, ((m, n), r) in enumerate(zip(shapes, ranks))]
    M = [torch.zeros(m, n, device=DEV) for m, n in shapes]
    return M, G, Q, W


@pytest.mark.parametrize("mode", ["colnorm", "qr"])
def test_ragged_ranks_equal_separate_calls(mode):
    # rank 0 = every matrix's rank from its Q_state rows; one ragged call must
    # give, bit for bit, what one call per matrix gives (ranks on both sides
    # of the one-CTA / blocked Cholesky threshold)
    shapes = [(256, 384), (512, 256), (300, 700), (640, 512)]
    ranks = [16, 48, 96, 300]
    M1, G, Q1, W1 = _state(shapes, ranks)
    M2, _, Q2, W2 = _state(shapes, ranks)
    sig1 = torch.empty(sum(ranks), device=DEV)
    sig2 = torch.empty(sum(ranks), device=DEV)
    p0 = ouo.dion_params(rank=0, norm_mode=mode)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    for _ in range(2):
        ouo.dion_lowrank_step(M1, G, Q1, W1, p0, scale=[1.0, 2.0, 1.0, 0.5], status=st, sigma=sig1)
        off = 0
        for i, r in enumerate(ranks):
            pi = ouo.dion_params(rank=r, norm_mode=mode)
            ouo.dion_lowrank_step([M2[i]], [G[i]], [Q2[i]], [W2[i]], pi,
                                  scale=[[1.0, 2.0, 1.0, 0.5][i]], status=st,
                                  sigma=sig2[off:off + r])
            off += r
    torch.cuda.synchronize()
    assert st.item() == 0
    for a, b in zip(M1 + Q1 + W1, M2 + Q2 + W2):
        assert torch.equal(a, b)
    assert torch.equal(sig1, sig2)


@pytest.mark.parametrize("mode", [odion.COLNORM, odion.QR])
def test_sigma_and_effective_rank_against_oracle(mode):
    m, n, r = 512, 768, 64
    G = synth.lowrank_plus_noise(m, n, 24, 0.02, 31, torch.bfloat16, DEV)
    M = torch.zeros(m, n, device=DEV)
    W = torch.zeros(m, n, device=DEV)
    q0 = _q0(n, r, 3)
    Qt = torch.tensor(q0.T.copy(), device=DEV)
    sig = torch.empty(r, device=DEV)
    p = ouo.dion_params(rank=r, norm_mode="qr" if mode == odion.QR else "colnorm")
    Mr, Qr = np.zeros((m, n), np.float32), q0.astype(np.float64)
    for _ in range(3):
        ouo.dion_lowrank_step([M], [G], [Qt], [W], p, sigma=sig)
        er = ouo.dion_effective_rank(sig, [r])
        torch.cuda.synchronize()
        ref = odion.dion_step(Mr, to64(G), Qr, np.zeros((m, n)), 0.95, 0.01, 1.0, mode)
        Mr, Qr = ref["M"], ref["Q"]
        s_gpu = sig.double().cpu().numpy()
        assert rel_fro(s_gpu, ref["sigma"]) <= TOL_BF16
        # the kernel's entropy matches the oracle's formula on the same sigma
        assert abs(er.item() - odion.effective_rank(s_gpu)) <= 1e-5 * odion.effective_rank(s_gpu)
        assert abs(er.item() - odion.effective_rank(ref["sigma"])) <= TOL_BF16 * r
        assert 1.0 <= er.item() <= r


def test_effective_rank_closed_forms_on_device():
    ranks = [37, 3, 4, 5]
    sig = torch.cat([torch.ones(37), torch.tensor([0.0, 3.0, 0.0]),
                     torch.tensor([2.0, 2.0, 0.0, 0.0]), torch.zeros(5)]).to(DEV)
    er = ouo.dion_effective_rank(sig, ranks).cpu().numpy()
    assert er[0] == pytest.approx(37.0, rel=1e-6)
    assert er[1] == pytest.approx(1.0, rel=1e-6)
    assert er[2] == pytest.approx(2.0, rel=1e-6)
    assert er[3] == 0.0


# ---- row-sharded step (the power iteration with rows spread over ranks) ---
def _full_state(m, n, r, seed, w_dtype=torch.float32):
    G = synth.lowrank_plus_noise(m, n, min(64, m, n), 0.02, seed, torch.bfloat16, DEV)
    W = synth.gaussian((m, n), seed + 7, 0.02, w_dtype, DEV)
    Q = torch.tensor(_q0(n, r, seed + 3).T.copy(), device=DEV)
    return torch.zeros(m, n, device=DEV), G, Q, W


@pytest.mark.parametrize("mode", ["colnorm", "qr"])
@pytest.mark.parametrize("r", [32, 128])
def test_shard_one_rank_is_the_unsharded_step(mode, r):
    m, n = 640, 512
    M1, G, Q1, W1 = _full_state(m, n, r, 11)
    M2, _, Q2, W2 = M1.clone(), None, Q1.clone(), W1.clone()
    p = ouo.dion_params(rank=r, norm_mode=mode, lr=0.05)
    step = ouo.DionShardStep([M2], [G], [Q2], [W2], p, rows_total=[m], scale=[1.5])
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    for _ in range(2):
        ouo.dion_lowrank_step([M1], [G], [Q1], [W1], p, scale=[1.5], status=st)
        step(lambda red: None, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    for a, b in ((M1, M2), (Q1, Q2), (W1, W2)):
        assert torch.equal(a, b)


@pytest.mark.parametrize("mode", [odion.COLNORM, odion.QR])
@pytest.mark.parametrize("splits", [(300, 340), (100, 260, 280)])
def test_shard_emulated_ranks_match_the_unsharded_step(mode, splits):
    # Ranks emulated in one process: each row block runs the four calls, and
    # between calls the blocks' partial sums are added (in rank order) and
    # handed back to every block -- what an all-reduce does.
    m, n, r = sum(splits), 512, 96
    name = "qr" if mode == odion.QR else "colnorm"
    M, G, Q, W = _full_state(m, n, r, 21)
    Mr, Wr = M.clone(), W.clone()
    W0 = to64(W)
    Qs = [Q.clone() for _ in splits]
    p = ouo.dion_params(rank=r, norm_mode=name, lr=0.05)
    bounds = np.concatenate([[0], np.cumsum(splits)]).astype(int)
    steps = [ouo.DionShardStep([Mr[a:b]], [G[a:b]], [Qs[k]], [Wr[a:b]], p, rows_total=[m])
             for k, (a, b) in enumerate(zip(bounds[:-1], bounds[1:]))]
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Mo, Qo, Wo = np.zeros((m, n), np.float32), _q0(n, r, 24).astype(np.float64), to64(W)
    for _ in range(2):
        for phase in ("project", "orth1", "orth2", "update"):
            for s_ in steps:
                getattr(s_, phase)(status=st)
            if phase != "update":
                tot = steps[0].red.clone()
                for s_ in steps[1:]:
                    tot += s_.red
                for s_ in steps:
                    s_.red.copy_(tot)
        ouo.dion_lowrank_step([M], [G], [Q], [W], p, status=st)
        ref = odion.dion_step(Mo, to64(G), Qo, Wo, 0.95, 0.05, 1.0, mode)
        Mo, Qo, Wo = ref["M"], ref["Q"], ref["W"]
    torch.cuda.synchronize()
    assert st.item() == 0
    for Qk in Qs[1:]:
        assert torch.equal(Qk, Qs[0])  # every rank forms the same right factor
    assert rel_fro(to64(Mr), to64(M)) <= 1e-2 and rel_fro(to64(Mr), Mo) <= TOL_BF16
    assert rel_fro(to64(Qs[0]), to64(Q)) <= 1e-2 and rel_fro(to64(Qs[0]).T, Qo) <= TOL_BF16
    assert rel_fro(to64(Wr) - W0, to64(W) - W0) <= 1e-2
