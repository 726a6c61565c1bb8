"""GPU parity of the batched Dion / Orth-Dion step on a mixed-shape batch.

Two layers of the Llama-3-8B-shaped parameter set (q, o 4096 x 4096; k, v
1024 x 4096; gate, up 14336 x 4096; down 4096 x 14336) step together in one
dion_lowrank_step call at rank 256, every operand of one shape laid out as
one evenly strided block so that each stage runs as grouped launches.
Sampled matrices of every shape are followed by the float64 oracle for three
steps, each side carrying its own state; one small matrix is also stepped
alone and must match its batched self bit for bit."""
import math

import numpy as np
import pytest
import torch

import orthonormalized_update_optimizers_b200 as ouo
from orthonormalized_update_optimizers_b200 import synth
from oracle import dion as odion

from ._util import TOL_BF16, rel_fro, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
R = 256
MU, LR = 0.95, 0.5


def _q0(n, r, seed):
    return odion.orth(synth.dion_q0(n, r, seed).double().numpy()).astype(np.float32)


@pytest.mark.parametrize("mode", [odion.COLNORM, odion.QR])
def test_two_llama8b_layers_batched_against_oracle(mode):
    shapes = [(m, n) for _, m, n in synth.llama8b_shapes(2)]
    names = [nm for nm, _, _ in synth.llama8b_shapes(2)]
    nmat = len(shapes)
    M = ouo.batch_empty(shapes, torch.float32, DEV)
    W = ouo.batch_empty(shapes, torch.bfloat16, DEV)
    Q = ouo.batch_empty([(R, n) for _, n in shapes], torch.float32, DEV)
    G = ouo.batch_empty(shapes, torch.bfloat16, DEV)
    for i, (m, n) in enumerate(shapes):
        G[i].copy_(synth.lowrank_plus_noise(m, n, 32, 0.01, synth.seed_for(3, i),
                                            torch.bfloat16, DEV))
        M[i].zero_()
        W[i].copy_(synth.gaussian((m, n), synth.seed_for(3, 1000 + i), 0.02,
                                  torch.bfloat16, DEV))
        Q[i].copy_(torch.from_numpy(_q0(n, R, 7 + i).T.copy()))
    scale = [math.sqrt(max(1.0, m / n)) for m, n in shapes]
    name = "qr" if mode == odion.QR else "colnorm"
    p = ouo.dion_params(rank=R, mu=MU, lr=LR, norm_mode=name)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    # one of every shape, both layers represented
    sample = [names.index(x) for x in ("layers.0.q", "layers.0.k", "layers.0.gate",
                                       "layers.1.down")]
    ref = {i: dict(M=np.zeros(shapes[i], np.float32), Q=_q0(shapes[i][1], R, 7 + i)
                   .astype(np.float64), W=to64(W[i])) for i in sample}
    G64 = {i: to64(G[i]) for i in sample}
    # the small sampled matrix alone, on copies of its state
    solo = names.index("layers.0.k")
    sM, sW, sQ = M[solo].clone(), W[solo].clone(), Q[solo].clone()
    Mb, Gb, Qb, Wb = ouo.MatBatch(M), ouo.MatBatch(G), ouo.MatBatch(Q), ouo.MatBatch(W)
    ws = torch.empty(ouo.dion_workspace_bytes(Mb, p), dtype=torch.uint8, device=DEV)
    for step in range(3):
        W_before = {i: to64(W[i]) for i in sample}
        ouo.dion_lowrank_step(Mb, Gb, Qb, Wb, p, scale=scale, workspace=ws, status=status)
        ouo.dion_lowrank_step([sM], [G[solo]], [sQ], [sW], p, scale=[scale[solo]],
                              status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        for i in sample:
            st = ref[i]
            out = odion.dion_step(st["M"], G64[i], st["Q"], st["W"], MU, LR, scale[i], mode)
            assert rel_fro(to64(M[i]), out["M"]) <= TOL_BF16, (step, names[i], "M")
            assert rel_fro(to64(Q[i]).T, out["Q"]) <= TOL_BF16, (step, names[i], "Q")
            # bf16 weights: the stored update carries one bf16 rounding of W
            W_after = to64(W[i])
            dW, dW_ref = W_after - W_before[i], out["W"] - st["W"]
            rnd = 2.0 ** -8 * np.linalg.norm(W_after)
            assert np.linalg.norm(dW_ref) > 4 * rnd  # the check has teeth
            e_w = max(0.0, np.linalg.norm(dW - dW_ref) - rnd) / np.linalg.norm(dW_ref)
            assert e_w <= TOL_BF16, (step, names[i], "W", e_w)
            st.update(M=out["M"], Q=out["Q"], W=out["W"])
        assert torch.equal(sM, M[solo]) and torch.equal(sQ, Q[solo])
        assert torch.equal(sW, W[solo])
