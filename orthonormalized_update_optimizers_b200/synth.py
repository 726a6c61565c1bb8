"""Seeded synthetic inputs shared by the CUDA path, its tests and the benchmark.

This module draws the gradient matrices, Dion's starting right factor and the
weights the optimizer step works on.  It holds none of the optimizer's own
arithmetic (no momentum, no Newton-Schulz, no row selection, no QR of the
method): it only makes random inputs of the shapes and spectra the workloads
describe, and both the GPU path and the float64 oracle consume the same bytes.

Workloads (sizes from the optimizer-step workloads this library is measured on):

* ``gaussian``: i.i.d. N(0, std^2) entries.
* ``lowrank_plus_noise``: ``U diag(s) V^T + N(0, noise^2)`` with ``U`` (m x r)
  and ``V`` (n x r) having orthonormal columns (QR of a Gaussian draw, a
  library routine used only for input synthesis) and ``s_i = i^(-1/2)``,
  i = 1..r.  A Gaussian gradient "plus a rank-r spike" is the same generator.

Seeds follow one rule: ``seed = 1000 * workload + matrix_index`` except the
single 256 x 1024 correctness matrix (seed 0) and Dion's starting factor
(seed 1).
"""
from __future__ import annotations

import torch

__all__ = [
    "gaussian",
    "lowrank_plus_noise",
    "dion_q0",
    "llama8b_shapes",
    "seed_for",
]


def seed_for(workload: int, index: int) -> int:
    """Seed of matrix ``index`` in workload number ``workload``."""
    return 1000 * int(workload) + int(index)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gaussian(shape, seed: int, std: float = 1.0, dtype=torch.float32,
             device="cpu") -> torch.Tensor:
    """N(0, std^2) entries drawn in fp32 from ``seed``, then cast to ``dtype``."""
    g = _gen(seed, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def lowrank_plus_noise(m: int, n: int, rank: int, noise_std: float, seed: int,
                       dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """``U diag(i^-1/2) V^T + N(0, noise_std^2)``, built in fp32, cast to ``dtype``.

    The low-rank factor's columns are orthonormalized with the library QR; this
    shapes the input spectrum only.
    """
    g = _gen(seed, device)
    r = max(0, min(int(rank), m, n))
    out = torch.randn(m, n, generator=g, device=device, dtype=torch.float32)
    out.mul_(noise_std)
    if r > 0:
        u = torch.randn(m, r, generator=g, device=device, dtype=torch.float32)
        v = torch.randn(n, r, generator=g, device=device, dtype=torch.float32)
        u = torch.linalg.qr(u, mode="reduced").Q
        v = torch.linalg.qr(v, mode="reduced").Q
        s = torch.arange(1, r + 1, device=device, dtype=torch.float32).rsqrt()
        out.addmm_(u * s, v.T)
    return out.to(dtype)


def dion_q0(n: int, r: int, seed: int = 1, device="cpu") -> torch.Tensor:
    """Dion's starting right factor: an n x r N(0,1) draw (fp32).

    The caller makes its columns orthonormal before the first step (the
    workloads orthonormalize it with the oracle's QR so that both sides start
    from identical bytes).
    """
    return gaussian((n, r), seed, 1.0, torch.float32, device)


def llama8b_shapes(n_layers: int = 32):
    """(name, rows, cols) of every 2-D weight of a Llama-3-8B-shaped model.

    Per layer: q, o 4096 x 4096; k, v 1024 x 4096; gate, up 14336 x 4096;
    down 4096 x 14336 (PyTorch ``[out, in]`` layout).
    """
    per_layer = [
        ("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096),
        ("o", 4096, 4096), ("gate", 14336, 4096), ("up", 14336, 4096),
        ("down", 4096, 14336),
    ]
    out = []
    for layer in range(n_layers):
        for name, m, n in per_layer:
            out.append((f"layers.{layer}.{name}", m, n))
    return out

