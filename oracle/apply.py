"""Weight update (oracle).

"Dion3：全栈正交更新", 输入输出流程: the step ends by updating the weights
with the orthogonalized block.  Reading (the pages give no formula): decoupled
weight decay then a scaled step,

    W[rows] <- (1 - lr * wd) * W[rows] - lr * scale * O

where ``rows`` are the kept rows (all rows when ``idx`` is None) and ``scale``
is a caller-chosen per-matrix factor.

TEST INFRASTRUCTURE: see the package docstring.
"""
from __future__ import annotations

import numpy as np


def apply_update(W, O, idx, lr: float, scale: float, wd: float = 0.0):
    """Return the updated weights in float64 (rows outside ``idx`` unchanged)."""
    W64 = np.asarray(W, dtype=np.float64).copy()
    O64 = np.asarray(O, dtype=np.float64)
    lr = float(np.float32(lr))
    scale = float(np.float32(scale))
    wd = float(np.float32(wd))
    decay = 1.0 - lr * wd
    if idx is None:
        W64 = decay * W64 - lr * scale * O64
    else:
        W64[idx] = decay * W64[idx] - lr * scale * O64
    return W64
