"""Oracle for the paged AdamW step of the LoRA parameters.

Test infrastructure only (see the package docstring). "QLoRA vs ChatGPT",
capability 4 and "Guanaco", "Core Architecture & Training" name paged
optimizers for the LoRA parameters but print no update rule; the reading is the
usual AdamW with decoupled weight decay and 32-bit moments, evaluated here in
fp64 from the fp32 state and the bf16 gradients:

    p <- p (1 - lr wd);  m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2
    p <- p - lr / (1 - b1^t) * m / (sqrt(v) / sqrt(1 - b2^t) + eps)
"""
from __future__ import annotations

import numpy as np


def adamw_step(p, g, m, v, step: int, lr: float, beta1: float, beta2: float, eps: float, weight_decay: float):
    """One AdamW step; every input is promoted exactly to fp64. Returns (p, m, v) in fp64."""
    f = lambda x: np.asarray(x, dtype=np.float64)  # noqa: E731
    p, g, m, v = f(p), f(g), f(m), f(v)
    lr, beta1, beta2, eps, weight_decay = (float(np.float32(x)) for x in (lr, beta1, beta2, eps, weight_decay))
    p = p * (1.0 - lr * weight_decay)
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    bc1 = 1.0 - beta1 ** step
    bc2 = 1.0 - beta2 ** step
    p = p - (lr / bc1) * m / (np.sqrt(v) / np.sqrt(bc2) + eps)
    return p, m, v
