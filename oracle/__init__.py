"""Float64 CPU oracle for the orthonormalized-update optimizer step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run anything in
this package.  The CUDA library and its Python binding never import it, and
the oracle imports nothing from them: the two share no code, no tables and no
helpers.  Both consume inputs from the seeded generator module
``orthonormalized_update_optimizers_b200.synth`` (which holds none of the
method's arithmetic).

Every function works one matrix at a time, in float64 (or in exact rationals
when handed ``fractions.Fraction`` object arrays), with library primitives only
for matrix products.  The sources it restates:

* "Dion3: Full-Stack Orthogonal Updates" (arXiv abstract): Muon's cubic-time
  Newton-Schulz step; Gram Newton-Schulz; orthogonalizing only a fraction of
  the momentum's rows.
* "Dion3：全栈正交更新" (ai-feeds summary), sections 核心洞察 / 核心模块 /
  输入输出流程 / 局限: Gram-NS on the symmetric Gram matrix with restarts and
  safety factors; the 1/8-of-rows rule with error feedback; the step order
  momentum -> row selection -> Gram-NS -> weight update.
* "Orth-Dion: Eliminating Geometric Mismatch in Distributed Low-Rank Spectral
  Optimization" (gist.science), sections Problem Statement, The Geometric
  Insight, Orth-Dion, Theoretical Contributions: Dion's single power-iteration
  step, residual buffer, column normalization versus QR.

Modules:

* ``momentum``  momentum update and the fp64 row keys.
* ``ns``        Frobenius normalization, quintic Newton-Schulz, Gram NS.
* ``dion3``     row selection, gather, error feedback, the full Dion3 step.
* ``dion``      Householder QR, column normalization, the Dion / Orth-Dion step,
                and ``effective_rank`` (a reading of Ada-Orth-Dion's estimator).
* ``apply``     the weight update.

Every function is pinned by tests under ``tests/`` to facts fixed by the pages
or by mathematics (closed forms through the SVD, exact rational equality,
brute force, invariants).  One exception: ``dion.effective_rank``, the
reading taken of Ada-Orth-Dion's entropy-based rank estimator, is pinned to
its own closed forms only.  The pages define no estimator, so its parity
with the method is unpinned.
"""
from . import apply, dion, dion3, momentum, ns  # noqa: F401

__all__ = ["apply", "dion", "dion3", "momentum", "ns"]
