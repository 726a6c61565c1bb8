"""The allocation-free Gram Newton-Schulz entry point.

gram_ns_orthogonalize_noalloc serves callers that cannot allocate device
memory (a plugin inside a framework whose pool owns all of it, or a path that
cannot afford cudaMalloc's implicit synchronization): it runs the same
kernels as gram_ns_orthogonalize with the library's fixed scratch array in
place of a caller workspace.  Both entry points run the same kernels in the
same order on the same inputs, and every reduction has a fixed order, so the
two results must agree bit for bit; the float64 oracle pins both.  This file
is collected last on purpose.
"""
import ctypes

import pytest
import torch

import orthonormalized_update_optimizers_b200 as ouo
from orthonormalized_update_optimizers_b200 import _lib as L
from orthonormalized_update_optimizers_b200 import synth
from oracle import ns as ons

from ._util import TOL_BF16, rel_fro, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _mats(tensors):
    arr = (L.OuoMat * len(tensors))()
    for i, t in enumerate(tensors):
        arr[i] = L.OuoMat(t.data_ptr(), t.shape[0], t.shape[1], t.stride(0))
    return arr


def _noalloc(X, O, p, status):
    s = torch.cuda.current_stream().cuda_stream
    return L.lib().gram_ns_orthogonalize_noalloc(
        _mats(X), L.OUO_BF16, _mats(O), L.OUO_BF16, len(X), ctypes.byref(p),
        status.data_ptr(), ctypes.c_void_p(s))


def test_noalloc_matches_workspace_entry_on_two_calls():
    p = ouo.ns_params()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    for call, (shape, seed) in enumerate([((256, 2048), 11), ((512, 1024), 12)]):
        X = [synth.lowrank_plus_noise(*shape, 64, 0.02, seed + i, torch.bfloat16, DEV)
             for i in range(2)]
        ref = [torch.empty_like(x) for x in X]
        ouo.gram_ns_orthogonalize(X, ref, p)            # caller workspace
        got = [torch.full_like(x, float("nan")) for x in X]
        assert _noalloc(X, got, p, status) == L.OUO_OK, L.lib().ouo_last_error()
        torch.cuda.synchronize()
        assert status.item() == 0
        for i, (g, r) in enumerate(zip(got, ref)):
            assert torch.equal(g, r), (call, i)
        # and both against the float64 oracle on the same bf16 inputs
        o = ons.gram_newton_schulz(to64(X[0]), iters=p.iters,
                                   restart_after=tuple(p.restart_after[:p.n_restart]))
        assert rel_fro(to64(got[0]), o) <= TOL_BF16, call


def test_noalloc_refuses_batches_beyond_its_array():
    p = ouo.ns_params()
    big = [torch.empty(2048, 8192, dtype=torch.bfloat16, device=DEV)]
    assert ouo.gram_ns_workspace_bytes(big, p) > L.OUO_NOALLOC_SCRATCH_BYTES
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    n0 = ouo.launch_count()
    rc = _noalloc(big, big, p, status)
    assert rc == L.OUO_ERR_WORKSPACE and b"scratch" in L.lib().ouo_last_error()
    assert ouo.launch_count() == n0  # nothing was launched


def test_noalloc_rejects_bad_parameters_before_sizing():
    # an unknown precision is an argument error, not a scratch-size refusal
    p = ouo.ns_params()
    p.precision = 7
    X = [torch.zeros(64, 128, dtype=torch.bfloat16, device=DEV)]
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    n0 = ouo.launch_count()
    assert _noalloc(X, X, p, status) == L.OUO_ERR_INVALID_ARG
    assert ouo.launch_count() == n0
