"""GPU parity of the Ada-Orth-Dion loop: the working rank of every matrix
follows the effective-rank estimate of the power iteration's singular-value
estimates, step after step, on a ragged batch.

Both sides apply the same host policy (ada.next_rank, ada.resize_state) to
their own estimates: the GPU to the sigma dion_lowrank_step writes and the
effective rank dion_effective_rank computes, the oracle to its own sigma and
effective_rank.  Growing states append the same seeded rows on both sides.
The chosen ranks must agree exactly, and M, Q and the weight update stay
within the bf16-path tolerance at every step.  The estimator itself is a
reading (the pages define none): its parity with the method is unpinned."""
import numpy as np
import pytest
import torch

import orthonormalized_update_optimizers_b200 as ouo
from orthonormalized_update_optimizers_b200 import ada, synth
from oracle import dion as odion

from ._util import TOL_BF16, rel_fro, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
MU, LR = 0.95, 0.05


def _q0(n, r, seed):
    return odion.orth(synth.dion_q0(n, r, seed).double().numpy()).astype(np.float32)


def test_ada_orth_dion_ranks_follow_the_estimate_on_both_sides():
    # (rows, cols, signal rank, starting rank): with slack 1.25 the working
    # rank of a spectrum sigma_i^2 ~ 1/i settles near 7 (k = 8, 16) and 10
    # (k = 12), inside the signal directions, so a shrinking state always
    # keeps directions with distinct sigma; the first and last states grow,
    # the second shrinks
    cfg = [(512, 1024, 16, 6), (384, 768, 12, 24), (256, 512, 8, 3)]
    r_min, r_max, slack = 2, 32, 1.25
    G = [synth.lowrank_plus_noise(m, n, k, 1e-3, 4000 + i, torch.bfloat16, DEV)
         for i, (m, n, k, _) in enumerate(cfg)]
    M = [torch.zeros(m, n, device=DEV) for m, n, _, _ in cfg]
    W = [synth.gaussian((m, n), 4100 + i, 0.02, torch.float32, DEV)
         for i, (m, n, _, _) in enumerate(cfg)]
    Q = [torch.tensor(_q0(n, r, 4200 + i).T.copy(), device=DEV)
         for i, (m, n, _, r) in enumerate(cfg)]
    ref = [dict(M=np.zeros((m, n), np.float32), Q=_q0(n, r, 4200 + i).astype(np.float64),
                W=to64(W[i])) for i, (m, n, _, r) in enumerate(cfg)]
    G64 = [to64(g) for g in G]
    p = ouo.dion_params(rank=0, mu=MU, lr=LR, norm_mode="qr")
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    history = []
    for step in range(6):
        ranks = [int(q.shape[0]) for q in Q]
        sig = torch.empty(sum(ranks), device=DEV)
        W_before = [to64(w) for w in W]
        ouo.dion_lowrank_step(M, G, Q, W, p, status=status, sigma=sig)
        er = ouo.dion_effective_rank(sig, ranks)
        torch.cuda.synchronize()
        assert status.item() == 0
        sig_h = sig.cpu().numpy()
        er_h = er.cpu().numpy()
        off = 0
        chosen = []
        for i, (m, n, _, _) in enumerate(cfg):
            r = ranks[i]
            st = ref[i]
            out = odion.dion_step(st["M"], G64[i], st["Q"], st["W"], MU, LR, 1.0, odion.QR)
            assert out["Q"].shape[1] == r
            assert rel_fro(to64(M[i]), out["M"]) <= TOL_BF16, (step, i, "M")
            assert rel_fro(to64(Q[i]).T, out["Q"]) <= TOL_BF16, (step, i, "Q")
            assert rel_fro(to64(W[i]) - W_before[i], out["W"] - st["W"]) <= TOL_BF16, (step, i)
            s_gpu = sig_h[off:off + r]
            off += r
            # the policy on each side's own estimate
            r_gpu = ada.next_rank(float(er_h[i]), r, r_min, r_max, slack=slack)
            r_ref = ada.next_rank(odion.effective_rank(out["sigma"]), r, r_min, r_max,
                                  slack=slack)
            assert r_gpu == r_ref, (step, i, float(er_h[i]), odion.effective_rank(out["sigma"]))
            chosen.append(r_gpu)
            # resize both states; growing appends the same seeded rows
            g1 = torch.Generator().manual_seed(7000 + 10 * step + i)
            g2 = torch.Generator().manual_seed(7000 + 10 * step + i)
            Q[i] = ada.resize_state(Q[i], [float(x) for x in s_gpu], r_gpu, generator=g1)
            q_ref = ada.resize_state(torch.from_numpy(out["Q"].T.copy()),
                                     [float(x) for x in out["sigma"]], r_ref, generator=g2)
            ref[i] = dict(M=out["M"], Q=q_ref.numpy().T.astype(np.float64), W=out["W"])
        history.append(chosen)
    # the ranks moved: the first state grew, the second shrank
    assert history[-1][0] > cfg[0][3] and history[-1][1] < cfg[1][3], history
    assert history[-1][2] > cfg[2][3], history
