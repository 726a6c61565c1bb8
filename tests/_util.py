"""Small helpers shared by the GPU parity tests (no method arithmetic)."""
import numpy as np
import torch


def to64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a CUDA/CPU tensor (bf16 and fp32 convert exactly)."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def bf16_round(x) -> np.ndarray:
    """Round float64 values to bf16 (nearest even) and back to float64."""
    t = torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.float().numpy().astype(np.float64)


# Tolerances stated for the orthogonalized outputs: relative Frobenius error
# against the float64 oracle.
TOL_BF16 = 2e-2
TOL_FP32 = 1e-4
