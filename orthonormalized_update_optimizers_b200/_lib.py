"""ctypes view of liborthoupd.so (the C ABI declared in include/orthoupd.h).

Only struct layouts, prototypes and the library handle live here.  Nothing in
this module computes anything; if the shared library is missing the first
call raises instead of falling back to any other implementation.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liborthoupd.so")

# ---- constants mirrored from include/orthoupd.h
OUO_OK = 0
OUO_ERR_INVALID_ARG = -1
OUO_ERR_UNSUPPORTED = -2
OUO_ERR_WORKSPACE = -3
OUO_ERR_CUDA = -4
OUO_ERR_NO_DEVICE = -5
OUO_F32 = 0
OUO_BF16 = 1
OUO_MOMENTUM_EMA = 0
OUO_MOMENTUM_ACCUM = 1
OUO_EF_NONE = 0
OUO_EF_ROWS = 1
OUO_PREC_BF16 = 0
OUO_PREC_FP32 = 1
OUO_DION_COLNORM = 0
OUO_DION_QR = 1
OUO_STATUS_TIMEOUT = 1
OUO_STATUS_BREAKDOWN = 2
OUO_MAX_RESTARTS = 8
OUO_NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024

# every symbol the header declares
EXPORTED = (
    "ouo_version", "ouo_last_error", "ouo_launch_count", "ouo_timing_enable",
    "ouo_timing_read", "ouo_debug_wait_timeout", "ouo_ns_default", "ouo_dion_default",
    "dion_momentum_update", "dion3_num_selected", "dion3_select_rows",
    "ns_workspace_bytes", "ns_orthogonalize", "gram_ns_workspace_bytes",
    "gram_ns_orthogonalize", "gram_ns_orthogonalize_noalloc", "apply_update",
    "dion_workspace_bytes", "dion_lowrank_step", "dion_workspace_bytes_ranks",
    "dion_lowrank_step_stats", "dion_effective_rank", "dion_shard_workspace_bytes",
    "dion_shard_red_floats", "dion_shard_project", "dion_shard_orth1", "dion_shard_orth2",
    "dion_shard_update",
)


class OuoMat(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("ld", ctypes.c_int64)]


class NsParams(ctypes.Structure):
    _fields_ = [("a", ctypes.c_float), ("b", ctypes.c_float),
                ("c", ctypes.c_float), ("iters", ctypes.c_int),
                ("safety", ctypes.c_float), ("eps", ctypes.c_float),
                ("normalize", ctypes.c_int), ("precision", ctypes.c_int),
                ("n_restart", ctypes.c_int),
                ("restart_after", ctypes.c_int * OUO_MAX_RESTARTS)]


class DionParams(ctypes.Structure):
    _fields_ = [("rank", ctypes.c_int), ("mu", ctypes.c_float),
                ("beta", ctypes.c_float), ("lr", ctypes.c_float),
                ("wd", ctypes.c_float), ("norm_mode", ctypes.c_int),
                ("eps", ctypes.c_float)]


class OuoError(RuntimeError):
    def __init__(self, func, code, msg):
        super().__init__(f"{func} failed ({code}): {msg}")
        self.code = code


_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_D = ctypes.c_double
_SZ = ctypes.c_size_t
_MP = ctypes.POINTER(OuoMat)
_NP = ctypes.POINTER(NsParams)
_DP = ctypes.POINTER(DionParams)
_I64 = ctypes.c_int64

_PROTOS = {
    "ouo_version": (_I, []),
    "ouo_last_error": (ctypes.c_char_p, []),
    "ouo_launch_count": (ctypes.c_ulonglong, []),
    "ouo_timing_enable": (_I, [_I]),
    "ouo_debug_wait_timeout": (_I, [_P, ctypes.c_ulonglong, _P]),
    "ouo_timing_read": (_I, [_I, ctypes.POINTER(ctypes.c_int),
                             ctypes.POINTER(ctypes.c_double),
                             ctypes.POINTER(ctypes.c_double)]),
    "ouo_ns_default": (None, [_NP]),
    "ouo_dion_default": (None, [_DP]),
    "dion_momentum_update": (_I, [_MP, _MP, _I, _I, _F, _I, _P, _P]),
    "dion3_num_selected": (_I64, [_I64, _D]),
    "dion3_select_rows": (_I, [_MP, _P, _I, _D, _I, _F, _F, _P, _MP, _I, _P, _P]),
    "ns_workspace_bytes": (_SZ, [_MP, _I, _NP]),
    "ns_orthogonalize": (_I, [_MP, _I, _MP, _I, _I, _NP, _P, _SZ, _P, _P]),
    "gram_ns_workspace_bytes": (_SZ, [_MP, _I, _NP]),
    "gram_ns_orthogonalize": (_I, [_MP, _I, _MP, _I, _I, _NP, _P, _SZ, _P, _P]),
    "gram_ns_orthogonalize_noalloc": (_I, [_MP, _I, _MP, _I, _I, _NP, _P, _P]),
    "apply_update": (_I, [_MP, _I, _MP, _I, _P, _I, _F, _P, _F, _P]),
    "dion_workspace_bytes": (_SZ, [_MP, _I, _DP]),
    "dion_lowrank_step": (_I, [_MP, _MP, _I, _MP, _MP, _I, _I, _DP, _P, _P, _SZ,
                               _P, _P]),
    "dion_workspace_bytes_ranks": (_SZ, [_MP, _P, _I, _DP]),
    "dion_lowrank_step_stats": (_I, [_MP, _MP, _I, _MP, _MP, _I, _I, _DP, _P, _P, _SZ,
                                     _P, _P, _P]),
    "dion_effective_rank": (_I, [_P, _P, _I, _P, _P]),
    "dion_shard_workspace_bytes": (_SZ, [_MP, _MP, _I, _DP]),
    "dion_shard_red_floats": (_SZ, [_MP, _MP, _I, _DP]),
    "dion_shard_project": (_I, [_MP, _MP, _I, _MP, _I, _DP, _P, _SZ, _P, _P, _P]),
    "dion_shard_orth1": (_I, [_MP, _MP, _I, _DP, _P, _P, _SZ, _P, _P, _P]),
    "dion_shard_orth2": (_I, [_MP, _MP, _I, _DP, _P, _P, _SZ, _P, _P, _P]),
    "dion_shard_update": (_I, [_MP, _MP, _MP, _I, _I, _DP, _P, _P, _SZ, _P, _P, _P]),
}


def lib():
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m orthonormalized_update_optimizers_b200.build` "
                "(there is no fallback implementation)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _PROTOS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def check(func: str, code: int) -> None:
    if code != OUO_OK:
        msg = lib().ouo_last_error()
        raise OuoError(func, code, msg.decode() if msg else "")
