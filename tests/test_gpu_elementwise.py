"""GPU parity of the HBM-bound kernels through the C ABI: momentum update
(+ float64 row keys), Dion3 row selection / gather / error feedback, and the
weight update, against the float64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import orthonormalized_update_optimizers_b200 as ouo
from orthonormalized_update_optimizers_b200 import synth
from oracle import apply as oapply
from oracle import dion3 as odion3
from oracle import momentum as omom

from ._util import rel_fro, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"

SHAPES = [(33, 70), (256, 1024), (128, 4096), (1, 8), (5, 3), (300, 129)]


def _pad_ld(t, extra):
    """Same values in a buffer whose row pitch is larger than the row."""
    m, n = t.shape
    big = torch.zeros(m, n + extra, dtype=t.dtype, device=t.device)
    big[:, :n] = t
    return big[:, :n]


@pytest.mark.parametrize("g_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("mode", ["ema", "accum"])
def test_momentum_update_batch(g_dtype, mode):
    Ms, Gs = [], []
    for i, (m, n) in enumerate(SHAPES):
        Ms.append(synth.gaussian((m, n), seed=100 + i, device=DEV))
        Gs.append(synth.gaussian((m, n), seed=200 + i, dtype=g_dtype, device=DEV))
    Ms[2] = _pad_ld(Ms[2], 4)  # ld > cols
    M0 = [to64(x) for x in Ms]
    total = sum(m for m, _ in SHAPES)
    keys = torch.empty(total, dtype=torch.float64, device=DEV)
    ouo.dion_momentum_update(Ms, Gs, 0.95, mode, keys)
    torch.cuda.synchronize()
    keys = keys.cpu().numpy()
    off = 0
    for i, (m, n) in enumerate(SHAPES):
        expect = omom.momentum_update(M0[i].astype(np.float32), to64(Gs[i]), 0.95,
                                      omom.EMA if mode == "ema" else omom.ACCUM)
        got = Ms[i].cpu().numpy()
        # fp32 state: single rounding of the exact update on both sides
        mism = np.count_nonzero(got != expect)
        assert mism <= max(1, got.size // 100000), (i, mism)
        assert np.allclose(got, expect, rtol=2e-7, atol=0)
        k_or = omom.row_sqnorms(got)
        assert np.max(np.abs(keys[off:off + m] - k_or) / np.maximum(k_or, 1e-300)) <= 1e-14
        off += m


def test_momentum_three_ema_steps_closed_form():
    G = synth.gaussian((256, 1024), seed=0, device=DEV)
    M = torch.zeros_like(G)
    for _ in range(3):
        ouo.dion_momentum_update([M], [G], 0.95, "ema")
    torch.cuda.synchronize()
    mu = float(np.float32(0.95))
    assert np.allclose(to64(M), (1 + mu + mu * mu) * to64(G), rtol=5e-7, atol=0)


def _keys_with_ties(m, seed):
    rng = np.random.default_rng(seed)
    base = rng.integers(0, 50, size=m).astype(np.float64)  # many exact ties
    base[rng.choice(m, size=max(1, m // 10), replace=False)] = 0.0
    return base


@pytest.mark.parametrize("rows,cols,rho", [(64, 96, 0.125), (1024, 256, 0.125),
                                           (1000, 72, 0.3), (7, 8, 1.0),
                                           (14336, 32, 0.125), (3, 5, 0.01)])
@pytest.mark.parametrize("ties", [False, True])
@pytest.mark.parametrize("x0_dtype", [torch.bfloat16, torch.float32])
def test_select_rows(rows, cols, rho, ties, x0_dtype):
    B = synth.gaussian((rows, cols), seed=rows + cols, device=DEV)
    if ties:
        keys64 = _keys_with_ties(rows, rows)
    else:
        keys64 = omom.row_sqnorms(to64(B))  # the stated key of the rows
    k = ouo.dion3_num_selected(rows, rho)
    assert k == odion3.num_selected(rows, rho)
    B0 = to64(B)
    keys = torch.tensor(keys64, dtype=torch.float64, device=DEV)
    idx = torch.empty(k, dtype=torch.int32, device=DEV)
    X0 = torch.empty(k, cols, dtype=x0_dtype, device=DEV)
    scale = torch.empty(1, dtype=torch.float32, device=DEV)
    ouo.dion3_select_rows([B], keys, rho, idx, [X0], scale, ef=True, mu=0.9)
    torch.cuda.synchronize()
    idx_or = odion3.select_rows(keys64, rho)
    assert np.array_equal(idx.cpu().numpy(), idx_or)  # bit-exact indices
    X0_or, factor = odion3.gather_normalize(B0, idx_or, keys64)
    assert scale.item() == pytest.approx(factor, rel=1e-6)
    x0 = to64(X0)
    if x0_dtype == torch.bfloat16:
        # one bf16 rounding on each side (<= 2^-9 relative each)
        assert np.all(np.abs(x0 - X0_or) <= 2.0 ** -8 * np.abs(X0_or) + 1e-30)
    else:
        assert rel_fro(x0, X0_or) <= 1e-6
    # error feedback: kept rows -> mu * B exactly (one fp32 rounding), others untouched
    Bn = B.cpu().numpy()
    expect = odion3.ef_write(B0, idx_or, 0.9)
    assert np.array_equal(Bn, expect)


def test_select_rows_batch_mixed_shapes():
    shapes = [(4096, 64), (1024, 64), (14336, 32), (4096, 128), (1024, 64)]
    Bs = [synth.gaussian(s, seed=300 + i, device=DEV) for i, s in enumerate(shapes)]
    B0 = [to64(b) for b in Bs]
    keys64 = np.concatenate([omom.row_sqnorms(b) for b in B0])
    keys = torch.tensor(keys64, device=DEV)
    ks = [ouo.dion3_num_selected(s[0], 0.125) for s in shapes]
    idx = torch.empty(sum(ks), dtype=torch.int32, device=DEV)
    X0 = [torch.empty(k, s[1], dtype=torch.bfloat16, device=DEV) for k, s in zip(ks, shapes)]
    scale = torch.empty(len(shapes), dtype=torch.float32, device=DEV)
    ouo.dion3_select_rows(Bs, keys, 0.125, idx, X0, scale, ef=False)
    torch.cuda.synchronize()
    off, koff = 0, 0
    for i, s in enumerate(shapes):
        idx_or = odion3.select_rows(keys64[off:off + s[0]], 0.125)
        assert np.array_equal(idx.cpu().numpy()[koff:koff + ks[i]], idx_or)
        assert np.array_equal(Bs[i].cpu().numpy(), B0[i].astype(np.float32))  # EF off
        off += s[0]
        koff += ks[i]


@pytest.mark.parametrize("w_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows_only", [False, True])
def test_apply_update(w_dtype, rows_only):
    shapes = [(64, 96), (33, 70), (512, 1024)]
    Ws = [synth.gaussian(s, seed=400 + i, dtype=w_dtype, device=DEV) for i, s in enumerate(shapes)]
    W0 = [to64(w) for w in Ws]
    idxs, Os = [], []
    for i, (m, n) in enumerate(shapes):
        if rows_only:
            k = ouo.dion3_num_selected(m, 0.25)
            sel = np.sort(np.random.default_rng(i).choice(m, k, replace=False)).astype(np.int32)
        else:
            sel = np.arange(m, dtype=np.int32)
        idxs.append(sel)
        Os.append(synth.gaussian((len(sel), n), seed=500 + i, dtype=torch.bfloat16, device=DEV))
    idx = torch.tensor(np.concatenate(idxs), device=DEV) if rows_only else None
    scale = [1.0, 0.5, 2.0]
    ouo.apply_update(Ws, Os, lr=0.02, idx=idx, scale=scale, wd=0.1)
    torch.cuda.synchronize()
    for i in range(len(shapes)):
        expect = oapply.apply_update(W0[i], to64(Os[i]), idxs[i] if rows_only else None,
                                     0.02, scale[i], 0.1)
        got = to64(Ws[i])
        if w_dtype == torch.float32:
            assert np.allclose(got, expect, rtol=1e-6, atol=1e-7)
        else:
            # one bf16 rounding of the fp32 result
            assert np.max(np.abs(got - expect) / np.maximum(np.abs(expect), 1e-3)) <= 2.0 ** -8
        if rows_only:
            untouched = np.setdiff1d(np.arange(shapes[i][0]), idxs[i])
            assert np.array_equal(got[untouched], W0[i][untouched])
