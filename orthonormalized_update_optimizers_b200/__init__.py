"""B200-native (sm_100a) orthonormalized-update optimizer step.

The hot path -- momentum update, Dion3 row selection, quintic and Gram
Newton-Schulz, Dion / Orth-Dion low-rank steps and the weight update -- runs
in hand-written CUDA kernels behind the C ABI of ``liborthoupd.so``
(``include/orthoupd.h``).  This package is the thin PyTorch binding: it
marshals tensors into that ABI and nothing else.
"""
from .binding import *  # noqa: F401,F403
from .binding import __all__ as _binding_all

__all__ = list(_binding_all)
