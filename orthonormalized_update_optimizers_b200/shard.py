"""Data-parallel partition of the Dion3 optimizer step across ranks.

Each weight matrix is an independent unit of the step: momentum, Dion3 row
selection and Gram Newton-Schulz touch one matrix at a time, and only the
weight update needs every matrix on every rank (data-parallel ranks keep a
full copy of the weights).  So the step is split by matrix:

  * every rank runs momentum, selection and Gram NS on its own matrices
    (its share of the momentum state lives on it alone);
  * the compressed updates -- per matrix the kept-row indices S (int32) and
    the orthonormalized block O (k x n, bf16) -- are all-gathered;
  * every rank applies every matrix's update to its copy of the weights.

This is the per-matrix partition with an all-gather of the updates that
"Dion3: Full-Stack Orthogonal Updates" (Abstract: megabatching reduces
communication overhead) and "Dion3：全栈正交更新" (核心模块: megabatching
compresses the data-parallel all-to-all) describe for sharded weights, in
its single-node form: the exchanged bytes are those of the k = ceil(rho m)
kept rows, a fraction rho of the dense update.

This module holds the host side: the partition plan (greedy longest-first
over an estimated per-matrix device time), and the byte layout of one
rank's exchange payload, so that selection writes S and Gram NS writes O
straight into the buffer the collective sends.  It computes nothing of the
method itself.
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import torch

ALIGN = 256  # byte alignment of every segment of a payload


def _align(x: int, a: int = ALIGN) -> int:
    return (x + a - 1) // a * a


def kept_rows(m: int, rho: float) -> int:
    """k = ceil(rho m), at least 1 and at most m (the Dion3 rule's count;
    the library's dion3_num_selected gives the same value)."""
    k = math.ceil(float(rho) * m - 1e-9)
    return max(1, min(m, k))


def matrix_cost(m: int, n: int, rho: float, hbm_gbs: float = 6500.0,
                bf16_tflops: float = 1300.0, tf32_tflops: float = 600.0) -> float:
    """Estimated device seconds of one matrix's share of the step: the
    HBM-bound momentum, gather and update passes plus the Gram NS products
    (5 iterations, one restart) on the k x n block at bf16 / tf32 rates."""
    k = kept_rows(m, rho)
    a, b = (k, n) if k <= n else (n, k)
    hbm = (10.0 * m * n + 8.0 * m + 10.0 * k * n + 6.0 * k * n) / (hbm_gbs * 1e9)
    bf = 2.0 * a * (a + 1) * b + 4.0 * a * a * b
    tf = 14.0 * a * a * (a + 1)
    return hbm + bf / (bf16_tflops * 1e12) + tf / (tf32_tflops * 1e12)


def plan_partition(shapes: Sequence[Tuple[int, int]], world: int,
                   rho: float) -> List[List[int]]:
    """Matrix indices per rank.  Longest-processing-time-first: matrices in
    decreasing estimated cost (ties: lower index first) go to the rank with
    the least accumulated cost (ties: lower rank).  Deterministic, so every
    rank computes the same plan.  Each rank's list is returned ascending."""
    if world < 1:
        raise ValueError("world must be >= 1")
    costs = [matrix_cost(m, n, rho) for m, n in shapes]
    order = sorted(range(len(shapes)), key=lambda i: (-costs[i], i))
    load = [0.0] * world
    parts: List[List[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda q: (load[q], q))
        parts[r].append(i)
        load[r] += costs[i]
    return [sorted(p) for p in parts]


class ExchangeLayout:
    """Byte layout of each rank's exchange payload.

    A rank's payload holds, at 256-byte aligned offsets: the int32 kept-row
    indices of all its matrices (concatenated in its matrix order, the
    layout dion3_select_rows and apply_update use), then each matrix's O
    block (k x n, bf16, row-major).  All payloads are padded to the largest
    one, so a single all-gather of `world * payload_bytes` bytes carries
    every update."""

    def __init__(self, shapes: Sequence[Tuple[int, int]], parts: Sequence[Sequence[int]],
                 rho: float):
        self.shapes = [(int(m), int(n)) for m, n in shapes]
        self.parts = [list(p) for p in parts]
        self.world = len(self.parts)
        self.k = [kept_rows(m, rho) for m, _ in self.shapes]
        self.idx_bytes = []
        self.o_off = []  # per rank: byte offset of each of its O blocks
        sizes = []
        for p in self.parts:
            ib = _align(4 * sum(self.k[i] for i in p))
            offs, pos = [], ib
            for i in p:
                offs.append(pos)
                pos += _align(2 * self.k[i] * self.shapes[i][1])
            self.idx_bytes.append(ib)
            self.o_off.append(offs)
            sizes.append(pos)
        self.payload_bytes = max(sizes) if sizes else 0
        self.used_bytes = sizes

    def views(self, buf: torch.Tensor, rank: int):
        """(idx, [O blocks]) of `rank`'s payload inside `buf`, a uint8 tensor
        of at least payload_bytes bytes (no copies)."""
        if buf.dtype != torch.uint8 or buf.dim() != 1 or buf.numel() < self.payload_bytes:
            raise ValueError("payload buffer must be a 1-D uint8 tensor of payload_bytes")
        p = self.parts[rank]
        nk = sum(self.k[i] for i in p)
        idx = buf[:4 * nk].view(torch.int32)
        blocks = []
        for i, off in zip(p, self.o_off[rank]):
            k, n = self.k[i], self.shapes[i][1]
            blocks.append(buf[off:off + 2 * k * n].view(torch.bfloat16).view(k, n))
        return idx, blocks

    def gathered_views(self, gathered: torch.Tensor):
        """Per source rank, the (idx, [O blocks]) views of an all-gathered
        buffer of world * payload_bytes bytes."""
        P = self.payload_bytes
        if gathered.numel() < self.world * P:
            raise ValueError("gathered buffer too small")
        return [self.views(gathered[r * P:(r + 1) * P], r) for r in range(self.world)]


def all_gather_payload(payload: torch.Tensor, gathered: torch.Tensor, group=None) -> None:
    """gathered[r * P:(r + 1) * P] = rank r's payload, on every rank (one
    collective; with one rank a copy-free no-op when `gathered` is
    `payload`)."""
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized():
        if gathered.data_ptr() != payload.data_ptr():
            gathered[:payload.numel()].copy_(payload)
        return
    world = dist.get_world_size(group)
    if world == 1:
        if gathered.data_ptr() != payload.data_ptr():
            gathered[:payload.numel()].copy_(payload)
        return
    P = payload.numel()
    dist.all_gather_into_tensor(gathered[:world * P], payload, group=group)
