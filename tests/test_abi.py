"""CPU checks of the C ABI: the library builds and loads, exports every
symbol the header declares, and its host-side logic (defaults, k = ceil(rho
m), argument validation, refusal without a GPU) behaves as documented.  No
kernel is launched here."""
import ctypes
import os
import re

import pytest

from orthonormalized_update_optimizers_b200 import _lib as L
from orthonormalized_update_optimizers_b200 import build as B
from oracle import dion3 as odion3

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "orthoupd.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.lib()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:[A-Za-z_][A-Za-z0-9_]*[\s*]+)+"
                       r"([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_six_calls():
    names = _declared_functions()
    for call in ("dion_momentum_update", "ns_orthogonalize",
                 "gram_ns_orthogonalize", "dion3_select_rows",
                 "dion_lowrank_step", "apply_update"):
        assert call in names


def test_library_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert names, "no declarations parsed"
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(L.EXPORTED) == sorted(names)


def test_version_and_defaults(lib):
    assert lib.ouo_version() == 1
    p = L.NsParams()
    lib.ouo_ns_default(ctypes.byref(p))
    assert (p.a, p.iters, p.normalize, p.n_restart, p.restart_after[0]) == (
        pytest.approx(3.4445), 5, 1, 1, 3)
    assert p.b == pytest.approx(-4.7750) and p.c == pytest.approx(2.0315)
    assert p.eps == pytest.approx(1e-7) and p.safety == 1.0
    d = L.DionParams()
    lib.ouo_dion_default(ctypes.byref(d))
    assert (d.rank, d.norm_mode) == (256, L.OUO_DION_COLNORM)
    assert d.mu == pytest.approx(0.95) and d.eps == pytest.approx(1e-8)


@pytest.mark.parametrize("m", [1, 2, 7, 8, 9, 100, 1000, 1001, 1024, 4096,
                               14336, 65537])
@pytest.mark.parametrize("rho", [1e-6, 0.1, 0.125, 0.3, 1 / 3, 0.5, 0.999, 1.0])
def test_num_selected_matches_oracle(lib, m, rho):
    assert lib.dion3_num_selected(m, rho) == odion3.num_selected(m, rho)


def test_num_selected_rejects_bad_input(lib):
    assert lib.dion3_num_selected(0, 0.5) == -1
    assert lib.dion3_num_selected(10, 0.0) == -1
    assert lib.dion3_num_selected(10, 1.5) == -1


def _mat(ptr, rows, cols, ld=None):
    return L.OuoMat(ptr, rows, cols, cols if ld is None else ld)


def test_validation_errors_before_any_launch(lib):
    # Bad arguments are refused on the host with OUO_ERR_INVALID_ARG and a
    # message; nothing is dereferenced (the pointers here are fake).
    arr = (L.OuoMat * 1)(_mat(None, 4, 8))
    g = (L.OuoMat * 1)(_mat(0x10000, 4, 8))
    rc = lib.dion_momentum_update(arr, g, 1, L.OUO_BF16, 0.9, 0, None, None)
    assert rc == -1 and b"NULL" in lib.ouo_last_error()
    m = (L.OuoMat * 1)(_mat(0x10002, 4, 8))  # not aligned to fp32
    rc = lib.dion_momentum_update(m, g, 1, L.OUO_BF16, 0.9, 0, None, None)
    assert rc == -1 and b"aligned" in lib.ouo_last_error()
    m = (L.OuoMat * 1)(_mat(0x10000, 4, 8, ld=6))  # ld < cols
    rc = lib.dion_momentum_update(m, g, 1, L.OUO_BF16, 0.9, 0, None, None)
    assert rc == -1
    m = (L.OuoMat * 1)(_mat(0x10000, 4, 9, ld=12))  # shape mismatch
    rc = lib.dion_momentum_update(m, g, 1, L.OUO_F32, 0.9, 0, None, None)
    assert rc == -1 and b"but" in lib.ouo_last_error()
    m = (L.OuoMat * 1)(_mat(0x10000, 4, 8))
    rc = lib.dion_momentum_update(m, g, 1, L.OUO_F32, 0.9, 7, None, None)
    assert rc == -1 and b"mode" in lib.ouo_last_error()
    # rho outside (0, 1]
    x0 = (L.OuoMat * 1)(_mat(0x20000, 1, 8))
    rc = lib.dion3_select_rows(m, 0x30000, 1, 1.5, 1, 0.9, 1e-7, 0x40000, x0,
                               L.OUO_BF16, 0x50000, None)
    assert rc == -1 and b"rho" in lib.ouo_last_error()
    # wrong X0 shape for k = ceil(rho m)
    rc = lib.dion3_select_rows(m, 0x30000, 1, 0.5, 1, 0.9, 1e-7, 0x40000, x0,
                               L.OUO_BF16, 0x50000, None)
    assert rc == -1 and b"X0" in lib.ouo_last_error()


def test_ns_workspace_and_params_validation(lib):
    x = (L.OuoMat * 2)(_mat(0x10000, 128, 512), _mat(0x20000, 300, 64))
    p = L.NsParams()
    lib.ouo_ns_default(ctypes.byref(p))
    a = lib.gram_ns_workspace_bytes(x, 2, ctypes.byref(p))
    b = lib.ns_workspace_bytes(x, 2, ctypes.byref(p))
    assert a > 0 and b > 0
    # workspace too small is refused before launching
    rc = lib.gram_ns_orthogonalize(x, L.OUO_BF16, x, L.OUO_BF16, 2,
                                   ctypes.byref(p), 0x100000, 16, None, None)
    assert rc == -3
    p.iters = -1
    rc = lib.gram_ns_orthogonalize(x, L.OUO_BF16, x, L.OUO_BF16, 2,
                                   ctypes.byref(p), 0x100000, 1 << 40, None,
                                   None)
    assert rc == -1
    p.iters = 5
    p.safety = 0.5
    rc = lib.ns_orthogonalize(x, L.OUO_BF16, x, L.OUO_BF16, 2,
                              ctypes.byref(p), 0x100000, 1 << 40, None, None)
    assert rc == -1 and b"safety" in lib.ouo_last_error()


def test_refuses_without_a_device(lib):
    # Valid arguments on a machine with no GPU: the call fails loudly
    # (OUO_ERR_NO_DEVICE) instead of computing anything elsewhere.
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    m = (L.OuoMat * 1)(_mat(0x10000, 4, 8))
    g = (L.OuoMat * 1)(_mat(0x20000, 4, 8))
    rc = lib.dion_momentum_update(m, g, 1, L.OUO_F32, 0.9, 0, None, None)
    assert rc == -5
