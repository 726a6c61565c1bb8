"""PyTorch-facing binding of liborthoupd.so: argument marshalling only.

Each function turns lists of 2-D CUDA tensors into ``ouo_mat`` arrays, picks
the current CUDA stream, calls the C entry point of the same name and raises
``OuoError`` on a nonzero return.  Every step of the optimizer runs inside the
library's kernels; there is no fallback.  Workspaces default to a torch
allocation made here (the library itself never allocates).
"""
from __future__ import annotations

import contextlib
import ctypes
from typing import Iterable, Optional, Sequence

import torch

from . import _lib as L
from ._lib import OuoError  # noqa: F401  (re-exported)

__all__ = [
    "MatBatch", "ns_params", "dion_params", "dion_momentum_update",
    "dion3_num_selected", "dion3_select_rows", "ns_workspace_bytes",
    "ns_orthogonalize", "gram_ns_workspace_bytes", "gram_ns_orthogonalize",
    "gram_ns_orthogonalize_noalloc",
    "apply_update", "dion_workspace_bytes", "dion_lowrank_step", "dion_effective_rank",
    "DionShardStep", "version",
    "launch_count", "timing_enable", "timing_read", "batch_empty", "check_vector",
]


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return L.OUO_F32
    if t.dtype == torch.bfloat16:
        return L.OUO_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def check_vector(t: Optional[torch.Tensor], name: str, dtype: torch.dtype,
                 numel: int, device: Optional[torch.device] = None) -> None:
    """The library reads and writes `numel` elements of `dtype` at
    t.data_ptr(): refuse anything else before the pointer reaches it (a wrong
    dtype or a short buffer would be a silent out-of-bounds access).  None
    passes (the optional arguments)."""
    if t is None:
        return
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() < numel:
        raise ValueError(f"{name} needs at least {numel} elements, got {t.numel()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the matrices on {device}")


class MatBatch:
    """A list of 2-D row-major CUDA tensors described once as an ouo_mat
    array, so repeated calls do not rebuild it.  All of them must live on
    one device."""

    def __init__(self, tensors: Iterable[torch.Tensor]):
        self.tensors = list(tensors)
        self.n = len(self.tensors)
        self.arr = (L.OuoMat * max(self.n, 1))()
        codes = set()
        for i, t in enumerate(self.tensors):
            if t.dim() != 2 or (t.shape[1] > 1 and t.stride(1) != 1):
                raise ValueError("every matrix must be 2-D with unit column stride")
            if not t.is_cuda:
                raise ValueError("every matrix must be a CUDA tensor")
            if t.device != self.tensors[0].device:
                raise ValueError("every matrix of a batch must be on one device")
            self.arr[i] = L.OuoMat(t.data_ptr(), t.shape[0], t.shape[1],
                                   max(t.stride(0), t.shape[1]))
            codes.add(_dtype_code(t))
        if len(codes) > 1:
            raise TypeError("a batch must have one dtype")
        self.dtype = codes.pop() if codes else L.OUO_F32

    @property
    def device(self):
        return self.tensors[0].device if self.tensors else torch.device("cuda")


def batch_empty(shapes: Sequence[Sequence[int]], dtype=torch.bfloat16,
                device=None) -> list:
    """Uninitialised matrices, one per (rows, cols) in ``shapes``, carved so
    that all matrices of one shape are consecutive slices of one contiguous
    [count, rows, cols] block, in the order they appear.  A Newton-Schulz
    input batch laid out this way (one uniform stride per shape) is read in
    place instead of being copied into the workspace first."""
    order = {}
    for s in shapes:
        order.setdefault((int(s[0]), int(s[1])), []).append(None)
    blocks = {key: torch.empty((len(v), key[0], key[1]), dtype=dtype, device=device)
              for key, v in order.items()}
    used = {key: 0 for key in order}
    out = []
    for s in shapes:
        key = (int(s[0]), int(s[1]))
        out.append(blocks[key][used[key]])
        used[key] += 1
    return out


def _batch(x) -> MatBatch:
    if isinstance(x, MatBatch):
        return x
    if isinstance(x, torch.Tensor):
        return MatBatch([x])
    return MatBatch(x)


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


@contextlib.contextmanager
def _on_device(*batches, stream=None, tensors=()):
    """Check that every matrix batch, extra tensor and the stream of one call
    live on one device, and make that device current for the call: the
    library launches on the current device and looks up per-device state
    there, so a call whose data sits on another GPU would hand that GPU's
    pointers to kernels on the wrong one."""
    dev = None
    for b in batches:
        if b is None or not b.tensors:
            continue
        if dev is None:
            dev = b.device
        elif b.device != dev:
            raise ValueError(f"a batch is on {b.device}, another on {dev}")
    for t in tensors:
        if t is None:
            continue
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"a buffer is on {t.device}, the matrices on {dev}")
    if stream is not None and dev is not None and stream.device != dev:
        raise ValueError(f"the stream is on {stream.device}, the matrices on {dev}")
    if dev is None:
        yield None
        return
    with torch.cuda.device(dev):
        yield dev


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def version() -> int:
    return L.lib().ouo_version()


def launch_count() -> int:
    """Kernels the library has enqueued in this process so far."""
    return int(L.lib().ouo_launch_count())


def timing_enable(on: bool = True) -> None:
    """Start (or stop and clear) event timing of tensor-core GEMM launches."""
    L.check("ouo_timing_enable", L.lib().ouo_timing_enable(1 if on else 0))


def timing_read(kind: int = -1):
    """(launches, total_ms, flops) of the recorded GEMM launches of one kind
    ((symmetric ? 4 : 0) + (tf32 ? 2 : 0) + (MN-major B ? 1 : 0); -1 = all)."""
    n = ctypes.c_int(0)
    ms = ctypes.c_double(0.0)
    fl = ctypes.c_double(0.0)
    L.check("ouo_timing_read", L.lib().ouo_timing_read(kind, ctypes.byref(n),
                                                      ctypes.byref(ms), ctypes.byref(fl)))
    return n.value, ms.value, fl.value


def ns_params(a=None, b=None, c=None, iters=None, safety=None, eps=None,
              normalize=None, precision="bf16", restart_after=None) -> L.NsParams:
    """ouo_ns_params with the library defaults, overridden where given."""
    p = L.NsParams()
    L.lib().ouo_ns_default(ctypes.byref(p))
    for name, val in (("a", a), ("b", b), ("c", c), ("iters", iters),
                      ("safety", safety), ("eps", eps)):
        if val is not None:
            setattr(p, name, val)
    if normalize is not None:
        p.normalize = int(bool(normalize))
    p.precision = {"bf16": L.OUO_PREC_BF16, "fp32": L.OUO_PREC_FP32}[precision]
    if restart_after is not None:
        ra = list(restart_after)
        if len(ra) > L.OUO_MAX_RESTARTS:
            raise ValueError("too many restarts")
        p.n_restart = len(ra)
        for i, t in enumerate(ra):
            p.restart_after[i] = int(t)
    return p


def dion_params(rank=None, mu=None, beta=None, lr=None, wd=None,
                norm_mode="colnorm", eps=None) -> L.DionParams:
    p = L.DionParams()
    L.lib().ouo_dion_default(ctypes.byref(p))
    for name, val in (("rank", rank), ("mu", mu), ("beta", beta), ("lr", lr),
                      ("wd", wd), ("eps", eps)):
        if val is not None:
            setattr(p, name, val)
    p.norm_mode = {"colnorm": L.OUO_DION_COLNORM, "qr": L.OUO_DION_QR}[norm_mode]
    return p


def _rows(b: MatBatch) -> int:
    return sum(int(t.shape[0]) for t in b.tensors)


def _dev(b: MatBatch) -> Optional[torch.device]:
    return b.tensors[0].device if b.tensors else None


def dion_momentum_update(M, G, mu: float, mode: str = "ema",
                         row_sqnorm: Optional[torch.Tensor] = None,
                         stream=None) -> None:
    Mb, Gb = _batch(M), _batch(G)
    check_vector(row_sqnorm, "row_sqnorm", torch.float64, _rows(Mb), _dev(Mb))
    code = {"ema": L.OUO_MOMENTUM_EMA, "accum": L.OUO_MOMENTUM_ACCUM}[mode]
    with _on_device(Mb, Gb, stream=stream):
        L.check("dion_momentum_update", L.lib().dion_momentum_update(
            Mb.arr, Gb.arr, Mb.n, Gb.dtype, mu, code, _ptr(row_sqnorm),
            _stream(stream)))


def dion3_num_selected(rows: int, rho: float) -> int:
    return int(L.lib().dion3_num_selected(rows, rho))


def dion3_select_rows(B, row_sqnorm: torch.Tensor, rho: float,
                      idx: torch.Tensor, X0, x0_scale: torch.Tensor,
                      ef: bool = True, mu: float = 0.95, eps: float = 1e-7,
                      stream=None) -> None:
    Bb, Xb = _batch(B), _batch(X0)
    if row_sqnorm is None or idx is None or x0_scale is None:
        raise ValueError("row_sqnorm, idx and x0_scale are required")
    nk = sum(dion3_num_selected(int(t.shape[0]), rho) for t in Bb.tensors)
    check_vector(row_sqnorm, "row_sqnorm", torch.float64, _rows(Bb), _dev(Bb))
    check_vector(idx, "idx", torch.int32, nk, _dev(Bb))
    check_vector(x0_scale, "x0_scale", torch.float32, Bb.n, _dev(Bb))
    with _on_device(Bb, Xb, stream=stream):
        L.check("dion3_select_rows", L.lib().dion3_select_rows(
            Bb.arr, _ptr(row_sqnorm), Bb.n, rho,
            L.OUO_EF_ROWS if ef else L.OUO_EF_NONE, mu, eps, _ptr(idx), Xb.arr,
            Xb.dtype, _ptr(x0_scale), _stream(stream)))


def ns_workspace_bytes(X, params=None) -> int:
    Xb = _batch(X)
    p = params or ns_params()
    return int(L.lib().ns_workspace_bytes(Xb.arr, Xb.n, ctypes.byref(p)))


def gram_ns_workspace_bytes(X, params=None) -> int:
    Xb = _batch(X)
    p = params or ns_params()
    return int(L.lib().gram_ns_workspace_bytes(Xb.arr, Xb.n, ctypes.byref(p)))


def _workspace(nbytes: int, device, given: Optional[torch.Tensor]):
    if given is not None:
        # an empty batch names no device index ("cuda"): check the rest only
        known = device if getattr(device, "index", None) is not None else None
        check_vector(given, "workspace", torch.uint8, nbytes, known)
        return given
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _run_ns(fname, wsfn, X, O, params, workspace, status, stream):
    Xb, Ob = _batch(X), _batch(O)
    p = params or ns_params()
    with _on_device(Xb, Ob, stream=stream):
        need = wsfn(Xb, p)
        ws = _workspace(need, Xb.device, workspace)
        check_vector(status, "status", torch.int32, 1, _dev(Xb))
        fn = getattr(L.lib(), fname)
        L.check(fname, fn(Xb.arr, Xb.dtype, Ob.arr, Ob.dtype, Xb.n, ctypes.byref(p),
                          ctypes.c_void_p(ws.data_ptr()), ws.numel(), _ptr(status),
                          _stream(stream)))


def ns_orthogonalize(X, O, params=None, workspace=None, status=None,
                     stream=None) -> None:
    _run_ns("ns_orthogonalize", ns_workspace_bytes, X, O, params, workspace,
            status, stream)


def gram_ns_orthogonalize(X, O, params=None, workspace=None, status=None,
                          stream=None) -> None:
    _run_ns("gram_ns_orthogonalize", gram_ns_workspace_bytes, X, O, params,
            workspace, status, stream)


def gram_ns_orthogonalize_noalloc(X, O, params=None, status=None,
                                  stream=None) -> None:
    """gram_ns_orthogonalize without a workspace, for callers that cannot
    allocate device memory: the library's fixed scratch array (shared by all
    calls; calls that overlap on the GPU race) stands in for it."""
    Xb, Ob = _batch(X), _batch(O)
    p = params or ns_params()
    check_vector(status, "status", torch.int32, 1, _dev(Xb))
    with _on_device(Xb, Ob, stream=stream):
        L.check("gram_ns_orthogonalize_noalloc", L.lib().gram_ns_orthogonalize_noalloc(
            Xb.arr, Xb.dtype, Ob.arr, Ob.dtype, Xb.n, ctypes.byref(p), _ptr(status),
            _stream(stream)))


def apply_update(W, O, lr: float, idx: Optional[torch.Tensor] = None,
                 scale: Optional[Sequence[float]] = None, wd: float = 0.0,
                 stream=None) -> None:
    Wb, Ob = _batch(W), _batch(O)
    check_vector(idx, "idx", torch.int32, _rows(Ob), _dev(Wb))
    sc = None
    if scale is not None:
        if len(scale) != Wb.n:
            raise ValueError("scale needs one value per matrix")
        sc = (ctypes.c_float * Wb.n)(*[float(s) for s in scale])
    with _on_device(Wb, Ob, stream=stream):
        L.check("apply_update", L.lib().apply_update(
            Wb.arr, Wb.dtype, Ob.arr, Ob.dtype, _ptr(idx), Wb.n, lr, sc, wd,
            _stream(stream)))


def _ranks(Mb, Qb, params):
    """Per-matrix ranks: params.rank, or each Q_state's row count when
    params.rank == 0 (ragged ranks)."""
    if params.rank:
        return [int(params.rank)] * Mb.n
    if Qb is None:
        raise ValueError("ragged ranks (rank=0) need the Q_state batch")
    return [int(t.shape[0]) for t in Qb.tensors]


def dion_workspace_bytes(M, params, Q_state=None) -> int:
    """Workspace bytes of dion_lowrank_step; with params.rank == 0 the ranks
    come from the Q_state batch (one rank per matrix)."""
    Mb = _batch(M)
    if params.rank:
        return int(L.lib().dion_workspace_bytes(Mb.arr, Mb.n, ctypes.byref(params)))
    Qb = _batch(Q_state) if Q_state is not None else None
    rk = (ctypes.c_int * max(Mb.n, 1))(*_ranks(Mb, Qb, params))
    return int(L.lib().dion_workspace_bytes_ranks(Mb.arr, rk, Mb.n, ctypes.byref(params)))


def dion_lowrank_step(M, G, Q_state, W, params, scale=None, workspace=None,
                      status=None, stream=None, sigma: Optional[torch.Tensor] = None) -> None:
    """One Dion / Orth-Dion step per matrix.  params.rank == 0 takes each
    matrix's rank from its Q_state rows.  With `sigma` (a float32 CUDA
    tensor of sum(ranks) elements) the step also writes the norms of R's
    columns, matrix after matrix."""
    Mb, Gb, Qb, Wb = _batch(M), _batch(G), _batch(Q_state), _batch(W)
    sc = None
    if scale is not None:
        if len(scale) != Mb.n:
            raise ValueError("scale needs one value per matrix")
        sc = (ctypes.c_float * Mb.n)(*[float(s) for s in scale])
    check_vector(sigma, "sigma", torch.float32, sum(_ranks(Mb, Qb, params)), _dev(Mb))
    check_vector(status, "status", torch.int32, 1, _dev(Mb))
    with _on_device(Mb, Gb, Qb, Wb, stream=stream):
        need = dion_workspace_bytes(Mb, params, Qb)
        ws = _workspace(need, Mb.device, workspace)
        L.check("dion_lowrank_step", L.lib().dion_lowrank_step_stats(
            Mb.arr, Gb.arr, Gb.dtype, Qb.arr, Wb.arr, Wb.dtype, Mb.n,
            ctypes.byref(params), sc, ctypes.c_void_p(ws.data_ptr()), ws.numel(),
            _ptr(sigma), _ptr(status), _stream(stream)))


def dion_effective_rank(sigma: torch.Tensor, ranks: Sequence[int],
                        erank: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Per matrix exp(Shannon entropy of sigma_j^2 / sum sigma^2), from the
    sigma that dion_lowrank_step writes; returns a float32 CUDA tensor."""
    n = len(ranks)
    check_vector(sigma, "sigma", torch.float32, sum(int(r) for r in ranks))
    if erank is None:
        erank = torch.empty(max(n, 1), dtype=torch.float32, device=sigma.device)
    check_vector(erank, "erank", torch.float32, n, sigma.device)
    rk = (ctypes.c_int * max(n, 1))(*[int(r) for r in ranks])
    with _on_device(stream=stream, tensors=(sigma, erank)):
        L.check("dion_effective_rank", L.lib().dion_effective_rank(
            _ptr(sigma), rk, n, _ptr(erank), _stream(stream)))
    return erank


class DionShardStep:
    """The row-sharded Dion / Orth-Dion step of one rank: its row blocks of
    M, G, W for every matrix and a full copy of each Q_state.  The four
    library calls run in order; `allreduce(red)` must sum the float32 CUDA
    tensor `red` over the ranks in place (e.g. torch.distributed.all_reduce)
    and is called between them.  `rows_total` are the matrices' global row
    counts."""

    def __init__(self, M, G, Q_state, W, params, rows_total: Sequence[int], scale=None):
        self.Mb, self.Gb, self.Qb, self.Wb = _batch(M), _batch(G), _batch(Q_state), _batch(W)
        self.p = params
        n = self.Mb.n
        if len(rows_total) != n:
            raise ValueError("rows_total needs one entry per matrix")
        self.rows = (ctypes.c_int64 * max(n, 1))(*[int(x) for x in rows_total])
        if scale is not None and len(scale) != n:
            raise ValueError("scale needs one value per matrix")
        self.scale = None if scale is None else (ctypes.c_float * n)(*[float(x) for x in scale])
        self._check_devices()
        lib = L.lib()
        wsb = lib.dion_shard_workspace_bytes(self.Mb.arr, self.Qb.arr, n, ctypes.byref(params))
        rf = lib.dion_shard_red_floats(self.Mb.arr, self.Qb.arr, n, ctypes.byref(params))
        if n and (wsb == 0 or rf == 0):
            raise ValueError("invalid sharded Dion batch")
        dev = self.Mb.device
        self.ws = torch.empty(max(wsb, 256), dtype=torch.uint8, device=dev)
        self.red = torch.empty(max(rf, 64), dtype=torch.float32, device=dev)

    def _check_devices(self):
        with _on_device(self.Mb, self.Gb, self.Qb, self.Wb):
            pass

    def _args(self, status, stream):
        check_vector(status, "status", torch.int32, 1, self.red.device)
        if stream is not None and stream.device != self.red.device:
            raise ValueError(f"the stream is on {stream.device}, the matrices on "
                             f"{self.red.device}")
        with torch.cuda.device(self.red.device):
            return (ctypes.byref(self.p), ctypes.c_void_p(self.ws.data_ptr()),
                    self.ws.numel(), _ptr(self.red), _ptr(status), _stream(stream))

    def project(self, status=None, stream=None) -> None:
        pp, ws, wn, red, st, s = self._args(status, stream)
        L.check("dion_shard_project", L.lib().dion_shard_project(
            self.Mb.arr, self.Gb.arr, self.Gb.dtype, self.Qb.arr, self.Mb.n, pp, ws, wn,
            red, st, s))

    def orth1(self, status=None, stream=None) -> None:
        pp, ws, wn, red, st, s = self._args(status, stream)
        L.check("dion_shard_orth1", L.lib().dion_shard_orth1(
            self.Mb.arr, self.Qb.arr, self.Mb.n, pp, self.rows, ws, wn, red, st, s))

    def orth2(self, status=None, stream=None) -> None:
        pp, ws, wn, red, st, s = self._args(status, stream)
        L.check("dion_shard_orth2", L.lib().dion_shard_orth2(
            self.Mb.arr, self.Qb.arr, self.Mb.n, pp, self.rows, ws, wn, red, st, s))

    def update(self, status=None, stream=None) -> None:
        pp, ws, wn, red, st, s = self._args(status, stream)
        L.check("dion_shard_update", L.lib().dion_shard_update(
            self.Mb.arr, self.Qb.arr, self.Wb.arr, self.Wb.dtype, self.Mb.n, pp, self.scale,
            ws, wn, red, st, s))

    def __call__(self, allreduce, status=None, stream=None) -> None:
        """One step: the four calls with allreduce(self.red) between them."""
        self.project(status, stream)
        allreduce(self.red)
        self.orth1(status, stream)
        allreduce(self.red)
        self.orth2(status, stream)
        allreduce(self.red)
        self.update(status, stream)
