"""GPU parity of the whole Dion3 step (momentum -> row selection -> Gram NS
-> weight update) through the C ABI against the oracle's dion3_step."""
import numpy as np
import pytest
import torch

import orthonormalized_update_optimizers_b200 as ouo
from orthonormalized_update_optimizers_b200 import synth
from oracle import dion3 as odion3

from ._util import TOL_BF16, rel_fro, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run_gpu_step(Ms, Gs, Ws, rho, mu, lr, scales, ef=True, gram=True):
    total = sum(M.shape[0] for M in Ms)
    keys = torch.empty(total, dtype=torch.float64, device=DEV)
    ouo.dion_momentum_update(Ms, Gs, mu, "accum" if ef else "ema", keys)
    ks = [ouo.dion3_num_selected(M.shape[0], rho) for M in Ms]
    idx = torch.empty(sum(ks), dtype=torch.int32, device=DEV)
    X0 = [torch.empty(k, M.shape[1], dtype=torch.bfloat16, device=DEV) for k, M in zip(ks, Ms)]
    scale = torch.empty(len(Ms), dtype=torch.float32, device=DEV)
    ouo.dion3_select_rows(Ms, keys, rho, idx, X0, scale, ef=ef, mu=mu)
    O = [torch.empty_like(x) for x in X0]
    fn = ouo.gram_ns_orthogonalize if gram else ouo.ns_orthogonalize
    fn(X0, O, ouo.ns_params(normalize=False))
    ouo.apply_update(Ws, O, lr, idx=idx, scale=scales)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), ks, O


@pytest.mark.parametrize("ef", [True, False])
@pytest.mark.parametrize("gram", [True, False])
def test_dion3_step_lowrank_batch(ef, gram):
    # 4 matrices of 1024 x 4096 from the low-rank(64) + N(0, 0.02^2)
    # generator, fp32 momentum, rho = 1/8, Gram NS 5 iterations 1 restart.
    shapes = [(1024, 4096)] * 3 + [(512, 1024)]
    Gs = [synth.lowrank_plus_noise(m, n, 64, 0.02, synth.seed_for(1, i), torch.bfloat16, DEV)
          for i, (m, n) in enumerate(shapes)]
    Ms = [0.1 * synth.gaussian(s, 50 + i, 0.01, torch.float32, DEV) for i, s in enumerate(shapes)]
    Ws = [synth.gaussian(s, 60 + i, 0.02, torch.float32, DEV) for i, s in enumerate(shapes)]
    M0 = [to64(M) for M in Ms]
    W0 = [to64(W) for W in Ws]
    G64 = [to64(G) for G in Gs]
    scales = [1.0, 2.0, 0.5, 1.0]
    idx, ks, O = _run_gpu_step(Ms, Gs, Ws, 0.125, 0.95, 0.02, scales, ef, gram)
    off = 0
    for i in range(len(shapes)):
        ref = odion3.dion3_step(M0[i].astype(np.float32), G64[i], W0[i], 0.95, 0.125,
                                0.02, scales[i], ef_mode=odion3.EF_ROWS if ef else odion3.EF_NONE,
                                variant="gram" if gram else "std")
        assert np.array_equal(idx[off:off + ks[i]], ref["idx"])
        assert rel_fro(to64(O[i]), ref["O"]) <= TOL_BF16
        Mg = Ms[i].cpu().numpy()
        assert np.count_nonzero(Mg != ref["M"]) <= Mg.size // 100000 + 1
        dW = to64(Ws[i]) - W0[i]
        dW_ref = ref["W"] - W0[i]
        assert rel_fro(dW, dW_ref) <= TOL_BF16
        off += ks[i]


def test_dion3_repeated_steps_stay_close():
    # three consecutive steps on the same state: selections keep matching
    shape = (1024, 2048)
    M = torch.zeros(shape, dtype=torch.float32, device=DEV)
    W = torch.zeros(shape, dtype=torch.float32, device=DEV)
    Mr = np.zeros(shape, dtype=np.float32)
    Wr = np.zeros(shape)
    for step in range(3):
        G = synth.lowrank_plus_noise(*shape, 64, 0.02, 9000 + step, torch.bfloat16, DEV)
        idx, ks, O = _run_gpu_step([M], [G], [W], 0.125, 0.95, 0.01, [1.0])
        ref = odion3.dion3_step(Mr, to64(G), Wr, 0.95, 0.125, 0.01, 1.0)
        assert np.array_equal(idx, ref["idx"])
        assert rel_fro(to64(O[0]), ref["O"]) <= TOL_BF16
        # carry the oracle's own state forward (teacher-free: it never sees GPU values)
        Mr, Wr = ref["M"], ref["W"]
