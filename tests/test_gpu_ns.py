"""GPU parity of standard and Gram Newton-Schulz through the C ABI against
the float64 oracle on the same input bytes: bf16 tensor-core path within
2e-2 relative Frobenius error, fp32 path within 1e-4."""
import numpy as np
import pytest
import torch

import orthonormalized_update_optimizers_b200 as ouo
from orthonormalized_update_optimizers_b200 import synth
from oracle import ns as ons

from ._util import TOL_BF16, TOL_FP32, rel_fro, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(shape, dtype, seed, kind="lowrank"):
    m, n = shape
    if kind == "gauss":
        return synth.gaussian(shape, seed, 1.0, dtype, DEV)
    return synth.lowrank_plus_noise(m, n, min(64, m, n), 0.02, seed, dtype, DEV)


def _oracle(X64, gram, iters=5, safety=1.0, restarts=(3,), normalize=True):
    if gram:
        return ons.gram_newton_schulz(X64, iters, safety=safety, normalize=normalize,
                                      restart_after=restarts)
    return ons.newton_schulz(X64, iters, safety=safety, normalize=normalize)


CASES = [(33, 70), (128, 512), (256, 1024), (300, 128), (129, 1000), (512, 512),
         (1, 64), (64, 1), (8, 16)]


@pytest.mark.parametrize("gram", [True, False])
@pytest.mark.parametrize("precision", ["bf16", "fp32"])
@pytest.mark.parametrize("shape", CASES)
def test_ns_single(gram, precision, shape):
    dtype = torch.bfloat16 if precision == "bf16" else torch.float32
    X = _inputs(shape, dtype, seed=sum(shape))
    O = torch.empty_like(X)
    p = ouo.ns_params(precision=precision)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    fn = ouo.gram_ns_orthogonalize if gram else ouo.ns_orthogonalize
    fn([X], [O], p, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = _oracle(to64(X), gram)
    err = rel_fro(to64(O), ref)
    tol = TOL_BF16 if precision == "bf16" else TOL_FP32
    assert err <= tol, err


@pytest.mark.parametrize("gram", [True, False])
def test_ns_batch_mixed_shapes_bf16(gram):
    shapes = [(128, 4096), (128, 4096), (256, 1024), (512, 4096), (96, 200), (128, 4096)]
    Xs = [_inputs(s, torch.bfloat16, seed=1000 + i) for i, s in enumerate(shapes)]
    Os = [torch.empty(s, dtype=torch.float32, device=DEV) for s in shapes]  # fp32 out
    fn = ouo.gram_ns_orthogonalize if gram else ouo.ns_orthogonalize
    fn(Xs, Os, ouo.ns_params())
    torch.cuda.synchronize()
    for X, O in zip(Xs, Os):
        err = rel_fro(to64(O), _oracle(to64(X), gram))
        assert err <= TOL_BF16, err


@pytest.mark.parametrize("restarts", [(), (1,), (2, 4), (3,)])
@pytest.mark.parametrize("safety", [1.0, 1.01])
def test_gram_restart_schedules_and_safety(restarts, safety):
    X = _inputs((256, 2048), torch.bfloat16, seed=7)
    O = torch.empty_like(X)
    p = ouo.ns_params(safety=safety, restart_after=restarts)
    ouo.gram_ns_orthogonalize([X], [O], p)
    torch.cuda.synchronize()
    ref = _oracle(to64(X), True, safety=safety, restarts=restarts)
    assert rel_fro(to64(O), ref) <= TOL_BF16


def test_gram_fp32_restart_schedules():
    X = _inputs((200, 600), torch.float32, seed=8)
    for restarts in [(), (1,), (2, 4)]:
        O = torch.empty_like(X)
        ouo.gram_ns_orthogonalize([X], [O], ouo.ns_params(precision="fp32",
                                                          restart_after=restarts))
        torch.cuda.synchronize()
        assert rel_fro(to64(O), _oracle(to64(X), True, restarts=restarts)) <= TOL_FP32


@pytest.mark.parametrize("iters", [0, 1, 2, 7])
@pytest.mark.parametrize("gram", [True, False])
def test_iteration_counts(iters, gram):
    X = _inputs((128, 640), torch.bfloat16, seed=9)
    O = torch.empty_like(X)
    fn = ouo.gram_ns_orthogonalize if gram else ouo.ns_orthogonalize
    fn([X], [O], ouo.ns_params(iters=iters, restart_after=(1,) if iters > 2 else ()))
    torch.cuda.synchronize()
    ref = _oracle(to64(X), gram, iters=iters, restarts=(1,) if iters > 2 else ())
    assert rel_fro(to64(O), ref) <= TOL_BF16


def test_normalize_off_and_aliasing():
    X = _inputs((256, 1024), torch.float32, seed=10)
    Xn = X / (X.norm() + 1e-7)
    Y = Xn.clone()
    ouo.gram_ns_orthogonalize([Y], [Y], ouo.ns_params(normalize=False, precision="fp32"))
    torch.cuda.synchronize()
    ref = _oracle(to64(Xn), True, normalize=False)
    assert rel_fro(to64(Y), ref) <= TOL_FP32


def test_correctness_matrix_256x1024_against_svd():
    # 256 x 1024 fp32 N(0, 1), seed 0; momentum 0.95 from zero over 3 steps;
    # both variants; compared with the oracle and with the SVD: same singular
    # vectors, singular values inside the 5-iteration band.
    G = synth.gaussian((256, 1024), seed=0, device=DEV)
    M = torch.zeros_like(G)
    for _ in range(3):
        ouo.dion_momentum_update([M], [G], 0.95, "ema")
    M64 = to64(M)
    U, s, Vt = np.linalg.svd(M64, full_matrices=False)
    for gram in (False, True):
        for precision, tol in (("fp32", TOL_FP32), ("bf16", TOL_BF16)):
            Xin = M if precision == "fp32" else M.to(torch.bfloat16)
            O = torch.empty(256, 1024, dtype=torch.float32, device=DEV)
            fn = ouo.gram_ns_orthogonalize if gram else ouo.ns_orthogonalize
            fn([Xin], [O], ouo.ns_params(precision=precision))
            torch.cuda.synchronize()
            out = to64(O)
            assert rel_fro(out, _oracle(to64(Xin), gram)) <= tol
            if precision == "fp32":
                D = U.T @ out @ Vt.T
                off = D - np.diag(np.diag(D))
                assert np.abs(off).max() <= 1e-4
                sv = np.diag(D)
                assert sv.min() >= 0.68 and sv.max() <= 1.2025


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
@pytest.mark.parametrize("restarts", [(3,), (), (1, 3)])
def test_gram_contiguous_batch_read_in_place(precision, restarts):
    # A batch carved by batch_empty (one uniform stride per shape) is read in
    # place when normalization is off; the result must equal, bit for bit, the
    # same batch given as separate tensors (which goes through the copy), and
    # the inputs must be left untouched.  Two restarts force the copy path.
    dtype = torch.bfloat16 if precision == "bf16" else torch.float32
    shapes = [(128, 512), (64, 1000), (128, 512), (300, 128), (64, 1000), (128, 512)]
    src = [_inputs(s, dtype, 40 + i) for i, s in enumerate(shapes)]
    src = [(x.float() / x.float().norm()).to(dtype) for x in src]  # normalization is off
    Xc = ouo.batch_empty(shapes, dtype, DEV)
    for x, s in zip(Xc, src):
        x.copy_(s)
    Xs = [s.clone() for s in src]
    p = ouo.ns_params(precision=precision, normalize=False, restart_after=restarts)
    Oc = [torch.empty_like(x) for x in Xc]
    Os = [torch.empty_like(x) for x in Xs]
    ouo.gram_ns_orthogonalize(Xc, Oc, p)
    ouo.gram_ns_orthogonalize(Xs, Os, p)
    torch.cuda.synchronize()
    for a, b, x, s in zip(Oc, Os, Xc, src):
        assert torch.equal(a, b)
        assert torch.equal(x, s)
    for i in (0, 3):
        ref = _oracle(to64(src[i]), True, restarts=restarts, normalize=False)
        tol = TOL_BF16 if precision == "bf16" else TOL_FP32
        assert rel_fro(to64(Oc[i]), ref) <= tol


def test_gram_contiguous_batch_output_over_input():
    # O written over its own input block (full aliasing): the in-place read is
    # refused, the copy path runs, and the result equals the separate-output run.
    shapes = [(128, 512)] * 4
    Xc = ouo.batch_empty(shapes, torch.bfloat16, DEV)
    for i, x in enumerate(Xc):
        y = _inputs((128, 512), torch.float32, 60 + i)
        x.copy_(y / y.norm())
    ref = [torch.empty_like(x) for x in Xc]
    p = ouo.ns_params(normalize=False)
    ouo.gram_ns_orthogonalize(Xc, ref, p)
    ouo.gram_ns_orthogonalize(Xc, Xc, p)
    torch.cuda.synchronize()
    for a, b in zip(Xc, ref):
        assert torch.equal(a, b)


@pytest.mark.parametrize("gram", [True, False])
def test_single_cta_and_cta_pair_tiles_agree(gram, monkeypatch):
    # Matrices taller than 128 rows run on CTA-pair tiles (256 x 256) by
    # default (K-major B); OUO_CTA_PAIR=0 selects single-CTA 128 x 256 tiles,
    # OUO_CTA_PAIR=2 puts the MN-major Q X products on pairs too.  All must
    # meet the oracle and agree with each other within half the bf16
    # tolerance.
    shapes = [(300, 1000), (512, 2048), (1792, 4096), (256, 256)]
    Xs = [_inputs(s, torch.bfloat16, 70 + i) for i, s in enumerate(shapes)]
    p = ouo.ns_params()
    fn = ouo.gram_ns_orthogonalize if gram else ouo.ns_orthogonalize
    outs = {}
    for mode in ("1", "0", "2"):
        monkeypatch.setenv("OUO_CTA_PAIR", mode)
        Os = [torch.empty_like(x) for x in Xs]
        fn(Xs, Os, p)
        torch.cuda.synchronize()
        outs[mode] = Os
    for i, x in enumerate(Xs):
        if i < 2:
            ref = _oracle(to64(x), gram)
            for mode in outs:
                assert rel_fro(to64(outs[mode][i]), ref) <= TOL_BF16
        assert rel_fro(to64(outs["1"][i]), to64(outs["0"][i])) <= 1e-2
        assert rel_fro(to64(outs["2"][i]), to64(outs["0"][i])) <= 1e-2


@pytest.mark.parametrize("gram", [True, False])
def test_upper_stored_symmetric_matrices_change_no_bits(gram, monkeypatch):
    # Upper-stored k x k matrices (the default on pair tiles) read the lower
    # blocks as the transposed upper blocks -- the very values full storage
    # mirrors there -- so the result must be bit-identical to full storage
    # (OUO_SYM_HALF=0).  k = 300 takes the per-chunk transposed loads, k = 512
    # the 4-D ones.
    shapes = [(300, 1000), (512, 2048), (1792, 4096)]
    Xs = [_inputs(s, torch.bfloat16, 90 + i) for i, s in enumerate(shapes)]
    fn = ouo.gram_ns_orthogonalize if gram else ouo.ns_orthogonalize
    outs = {}
    for mode in ("1", "0"):
        monkeypatch.setenv("OUO_SYM_HALF", mode)
        Os = [torch.empty_like(x) for x in Xs]
        fn(Xs, Os, ouo.ns_params())
        torch.cuda.synchronize()
        outs[mode] = Os
    for i, x in enumerate(Xs):
        assert torch.equal(outs["1"][i], outs["0"][i]), shapes[i]
    ref = _oracle(to64(Xs[0]), gram)
    assert rel_fro(to64(outs["1"][0]), ref) <= TOL_BF16


@pytest.mark.parametrize("gram", [True, False])
def test_four_d_operand_loads_change_no_bits(gram, monkeypatch):
    # An MN-major B stage on single-CTA tiles (Q X, B X) is one 4-D TMA load
    # when the columns split into whole 64-column chunks, else one load per
    # chunk (OUO_TMA_4D=0 forces the latter).  Both place the same bytes in
    # shared memory, so the results must be bit-identical.  n = 1000 leaves a
    # partial chunk and takes the per-chunk loads either way.
    shapes = [(512, 2048), (256, 4096), (300, 1000)]
    Xs = [_inputs(s, torch.bfloat16, 110 + i) for i, s in enumerate(shapes)]
    fn = ouo.gram_ns_orthogonalize if gram else ouo.ns_orthogonalize
    outs = {}
    for mode in ("1", "0"):
        monkeypatch.setenv("OUO_TMA_4D", mode)
        Os = [torch.empty_like(x) for x in Xs]
        fn(Xs, Os, ouo.ns_params())
        torch.cuda.synchronize()
        outs[mode] = Os
    for i in range(len(Xs)):
        assert torch.equal(outs["1"][i], outs["0"][i]), shapes[i]
    ref = _oracle(to64(Xs[0]), gram)
    assert rel_fro(to64(outs["1"][0]), ref) <= TOL_BF16
