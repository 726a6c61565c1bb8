"""Host side of the data-parallel partition of the Dion3 step (CPU, gloo).

The per-matrix work is done here by the float64 oracle (test-side only);
what is under test is the partition plan, the payload layout and the
all-gather of the compressed updates: after the exchange every rank must
hold every matrix's kept-row indices and O block, and every rank's weights
must equal those of one process that stepped all matrices itself."""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from orthonormalized_update_optimizers_b200 import shard, synth
from oracle import apply as oapply
from oracle import dion3 as odion3

RHO, MU, LR = 0.125, 0.95, 0.02
SHAPES = [(64, 128), (128, 64), (96, 256), (256, 128), (40, 72), (128, 128), (72, 200)]


def test_plan_covers_every_matrix_once_and_balances_the_8b_step():
    shapes = [(m, n) for _, m, n in synth.llama8b_shapes(32)]
    costs = [shard.matrix_cost(m, n, RHO) for m, n in shapes]
    for world in (1, 2, 3, 4, 8):
        parts = shard.plan_partition(shapes, world, RHO)
        assert len(parts) == world
        flat = sorted(i for p in parts for i in p)
        assert flat == list(range(len(shapes)))
        assert all(p == sorted(p) for p in parts)
        loads = [sum(costs[i] for i in p) for p in parts]
        # LPT: the heaviest rank exceeds the mean by less than one matrix
        assert max(loads) - sum(loads) / world <= max(costs) + 1e-12
        assert parts == shard.plan_partition(shapes, world, RHO)  # deterministic


def test_plan_edge_cases():
    assert shard.plan_partition([], 3, RHO) == [[], [], []]
    assert shard.plan_partition([(8, 8)], 2, RHO) == [[0], []]
    with pytest.raises(ValueError):
        shard.plan_partition([(8, 8)], 0, RHO)


def test_kept_rows_matches_the_oracle_rule():
    for m in (1, 7, 8, 9, 1023, 1024, 14336):
        for rho in (0.125, 0.3, 1.0):
            assert shard.kept_rows(m, rho) == odion3.num_selected(m, rho)


def test_layout_offsets_are_aligned_and_disjoint():
    parts = shard.plan_partition(SHAPES, 3, RHO)
    lay = shard.ExchangeLayout(SHAPES, parts, RHO)
    buf = torch.zeros(lay.payload_bytes, dtype=torch.uint8)
    for r in range(3):
        idx, blocks = lay.views(buf, r)
        assert idx.numel() == sum(lay.k[i] for i in parts[r])
        spans = [(0, 4 * idx.numel())]
        for i, off, b in zip(parts[r], lay.o_off[r], blocks):
            assert off % shard.ALIGN == 0
            assert tuple(b.shape) == (lay.k[i], SHAPES[i][1])
            spans.append((off, off + 2 * b.numel()))
        spans.sort()
        for (a0, a1), (b0, _) in zip(spans, spans[1:]):
            assert a1 <= b0
        assert spans[-1][1] <= lay.payload_bytes


def _inputs(i, m, n):
    G = synth.lowrank_plus_noise(m, n, 8, 0.01, 700 + i, torch.bfloat16, "cpu").double().numpy()
    W = synth.gaussian((m, n), 800 + i, 0.02, torch.float32, "cpu").double().numpy()
    M = synth.gaussian((m, n), 900 + i, 0.01, torch.float32, "cpu").numpy()
    return M, G, W


def _scale(m, n):
    return float(np.sqrt(max(1.0, m / n)))


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        parts = shard.plan_partition(SHAPES, world, RHO)
        lay = shard.ExchangeLayout(SHAPES, parts, RHO)
        payload = torch.zeros(lay.payload_bytes, dtype=torch.uint8)
        idx, blocks = lay.views(payload, rank)
        pos = 0
        for i, blk in zip(parts[rank], blocks):
            m, n = SHAPES[i]
            M, G, W = _inputs(i, m, n)
            res = odion3.dion3_step(M, G, W, MU, RHO, LR, _scale(m, n))
            k = len(res["idx"])
            idx[pos:pos + k] = torch.from_numpy(res["idx"].astype(np.int32))
            blk.copy_(torch.from_numpy(res["O"]).to(torch.bfloat16))
            pos += k
        gathered = torch.zeros(world * lay.payload_bytes, dtype=torch.uint8)
        shard.all_gather_payload(payload, gathered)
        # every rank applies every matrix's update to its full weights
        Ws = {}
        for r, (gidx, gblocks) in enumerate(lay.gathered_views(gathered)):
            pos = 0
            for i, blk in zip(parts[r], gblocks):
                m, n = SHAPES[i]
                _, _, W = _inputs(i, m, n)
                k = lay.k[i]
                S = gidx[pos:pos + k].numpy().astype(np.int64)
                pos += k
                Ws[i] = oapply.apply_update(W, blk.double().numpy(), S, LR, _scale(m, n))
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), **{str(i): w for i, w in Ws.items()})
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_exchange_reproduces_the_single_process_step(world):
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_worker, args=(world, _free_port(), d), nprocs=world, join=True)
        got = [np.load(os.path.join(d, f"rank{r}.npz")) for r in range(world)]
        for i, (m, n) in enumerate(SHAPES):
            M, G, W = _inputs(i, m, n)
            res = odion3.dion3_step(M, G, W, MU, RHO, LR, _scale(m, n))
            # the exchanged O is bf16: the reference applies the same rounding
            O16 = torch.from_numpy(res["O"]).to(torch.bfloat16).double().numpy()
            ref = oapply.apply_update(W, O16, res["idx"], LR, _scale(m, n))
            for r in range(world):
                assert np.array_equal(got[r][str(i)], ref), (i, r)


# ---- row-sharded Dion step: the orchestration over gloo ranks -------------
from oracle import dion as odion  # noqa: E402
from orthonormalized_update_optimizers_b200.binding import DionShardStep  # noqa: E402


class _Float64Phases:
    """Test-side float64 stand-in for one rank's four library calls (the
    same decomposition: Gram matrices and P^T B are the only summed parts),
    so DionShardStep's orchestration can run over real gloo ranks."""

    def __init__(self, M, G, Qt, W, mu, lr, beta, mode, rows_total):
        self.M, self.G, self.Qt, self.W = M, G, Qt, W
        # the oracle takes mu and beta as the fp32 values the library receives
        self.mu, self.beta = float(np.float32(mu)), float(np.float32(beta))
        self.lr, self.mode = lr, mode
        self.r, self.n = Qt.shape
        self.red = torch.zeros(max(self.r * self.r, self.r * self.n), dtype=torch.float64)

    def _put(self, a):
        self.red.zero_()
        self.red[:a.size] = torch.from_numpy(np.ascontiguousarray(a).ravel())

    def _get(self, shape):
        return self.red[:shape[0] * shape[1]].numpy().reshape(shape).copy()

    def _chol_apply(self, Pt):
        S = self._get((self.r, self.r))
        Lc = np.linalg.cholesky(S)
        return np.linalg.solve(Lc, Pt)

    def project(self, status=None, stream=None):
        self.B = self.M + self.G
        self.Pt = self.Qt @ self.B.T
        self._put(self.Pt @ self.Pt.T)

    def orth1(self, status=None, stream=None):
        self.Pt = self._chol_apply(self.Pt)
        self._put(self.Pt @ self.Pt.T)

    def orth2(self, status=None, stream=None):
        self.Pt = self._chol_apply(self.Pt)
        self._put(self.Pt @ self.B)

    def update(self, status=None, stream=None):
        Rt = self._get((self.r, self.n))
        P = self.Pt.T
        self.M = self.beta * self.B - (self.beta - self.mu) * (P @ Rt)
        if self.mode == odion.QR:
            Qn = odion.orth(Rt.T).T
        else:
            Qn = (odion.colnorm(Rt.T)).T
        self.W = self.W - self.lr * (P @ Qn)
        self.Qt = Qn


def _shard_worker(rank, world, port, out_dir, mode):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m, n, r = 90, 40, 6
        rng = np.random.default_rng(5)
        G = rng.standard_normal((m, n))
        W = rng.standard_normal((m, n)) * 0.1
        Q0 = odion.orth(rng.standard_normal((n, r)))
        rows = np.array_split(np.arange(m), world)[rank]
        ph = _Float64Phases(np.zeros((len(rows), n)), G[rows], Q0.T.copy(), W[rows],
                            0.95, 0.1, 1.0, mode, m)
        for _ in range(2):
            DionShardStep.__call__(ph, lambda t: dist.all_reduce(t))
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), M=ph.M, W=ph.W, Q=ph.Qt, rows=rows)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", [odion.COLNORM, odion.QR])
def test_gloo_row_sharded_dion_matches_the_unsharded_oracle(mode):
    world = 3
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_shard_worker, args=(world, _free_port(), d, mode), nprocs=world, join=True)
        m, n, r = 90, 40, 6
        rng = np.random.default_rng(5)
        G = rng.standard_normal((m, n))
        W = rng.standard_normal((m, n)) * 0.1
        Q = odion.orth(rng.standard_normal((n, r)))
        M = np.zeros((m, n))
        for _ in range(2):
            ref = odion.dion_step(M, G, Q, W, 0.95, 0.1, 1.0, mode, state_dtype=None)
            M, Q, W = ref["M"], ref["Q"], ref["W"]
        for k in range(world):
            got = np.load(os.path.join(d, f"rank{k}.npz"))
            rows = got["rows"]
            assert np.allclose(got["M"], M[rows], rtol=0, atol=1e-9)
            assert np.allclose(got["W"], W[rows], rtol=0, atol=1e-9)
            assert np.allclose(got["Q"], Q.T, rtol=0, atol=1e-9)
