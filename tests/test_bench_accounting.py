"""CPU checks of the benchmark's accounting: the algorithmic flop counts it
divides by device time, the Dion byte count, and the traffic table it reads
from the committed profile summary.

The flop counts are checked against a count taken by running the oracle's
Gram Newton-Schulz with a matrix class that records every product, so the
bench's closed form and the iteration the pages describe ("Dion3: Full-Stack
Orthogonal Updates" and its summary, 核心模块: iterate on the Gram matrix,
restarts) cannot drift apart."""
import importlib.util
import os

import numpy as np

from oracle import ns as ons

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test",
                                                  os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class _Counted(np.ndarray):
    """ndarray whose matmuls are tallied by shape (symmetric k x k results
    and k x n results counted apart)."""
    log = []

    def __matmul__(self, other):
        out = np.matmul(np.asarray(self), np.asarray(other))
        _Counted.log.append((self.shape, np.shape(other)))
        return out.view(_Counted)

    def __rmatmul__(self, other):
        out = np.matmul(np.asarray(other), np.asarray(self))
        _Counted.log.append((np.shape(other), self.shape))
        return out.view(_Counted)


def _products(k, n, iters=5, restart_after=(3,)):
    rng = np.random.default_rng(0)
    X = rng.standard_normal((k, n)).view(_Counted)
    _Counted.log = []
    orig_prepare = ons._prepare

    def prepare(x, normalize, eps):
        x0, tr = orig_prepare(np.asarray(x), normalize, eps)
        return x0.view(_Counted), tr

    ons._prepare = prepare
    try:
        ons.gram_newton_schulz(X, iters=iters, restart_after=restart_after)
    finally:
        ons._prepare = orig_prepare
    return list(_Counted.log)


def test_gram_ns_flops_match_the_products_the_iteration_takes():
    b = _bench()
    k, n = 48, 160
    log = _products(k, n)
    # k x k results other than products with the identity (Q = I on a
    # segment's first iteration is not a product the kernels run)
    kk = [p for p in log if p[0] == (k, k) and p[1] == (k, k)]
    kn_sym = [p for p in log if p[0] == (k, n) and p[1] == (n, k)]   # X X^T
    kn = [p for p in log if p[0] == (k, k) and p[1] == (k, n)]       # Q X
    eye_products = 2  # H @ I at the first iteration of each segment
    bf, tf = b.gram_ns_flops(k, n)
    assert tf == (len(kk) - eye_products) * k * k * (k + 1)
    assert bf == len(kn_sym) * k * (k + 1) * n + len(kn) * 2 * k * k * n
    # the default schedule: 14 tf32 products, 2 Gram matrices, 2 Q X
    assert len(kk) - eye_products == 14 and len(kn_sym) == 2 and len(kn) == 2


def test_gram_ns_flops_orient_and_schedules():
    b = _bench()
    assert b.gram_ns_flops(300, 100) == b.gram_ns_flops(100, 300)
    # no restart: X X^T once, Q X once; 5 A^2, 4 H Q, 4 x 2 A updates
    bf, tf = b.gram_ns_flops(64, 256, restarts=())
    sym, syrk, qx = 64 * 64 * 65, 64 * 65 * 256, 2 * 64 * 64 * 256
    assert (bf, tf) == (syrk + qx, (5 + 4 + 8) * sym)


def test_step_flops_of_the_8b_set():
    # the figure the bench line reports as gram_ns.flops_tf32 / flops_bf16
    b = _bench()
    bf = tf = 0
    for _, m, n in b._workload_shapes(32):
        k = max(1, int(np.ceil(0.125 * m)))
        f = b.gram_ns_flops(k, n)
        bf += f[0]
        tf += f[1]
    assert tf == 5341620207616
    assert bf == 6212267540480


def test_dion_bytes_per_element():
    # B = M + G: read M 4, G 2, write B 4; two reads of B 8; the in-place
    # M update 8; the bf16 W update 4
    b = _bench()
    assert b.DION_BYTES_PER_ELEM == 10 + 8 + 8 + 4


def test_traffic_table_parses():
    # the summary's table has both rows the bench line may use, each with a
    # positive byte count and a 16-hex-digit source hash
    path = os.path.join(ROOT, "profiles", "launches_llama8b_dion3_gram_ns_step.md")
    rows = {}
    with open(path) as f:
        for line in f:
            parts = [p.strip() for p in line.strip().strip("|").split("|")]
            if len(parts) == 3 and parts[1].isdigit():
                rows[parts[0]] = (int(parts[1]), parts[2])
    assert set(rows) == {"umma_gemm_kernel tf32 symmetric", "momentum_kernel"}
    for nbytes, digest in rows.values():
        assert nbytes > 0 and len(digest) == 16
        int(digest, 16)
