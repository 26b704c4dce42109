"""Oracle for the QLoRA linear layer, forward and backward (fp64).

Test infrastructure only (see the package docstring).

Passages followed:
* "QLoRA vs ChatGPT", capability 2: a rank-r LoRA adapter (A, B) is trained on
  top of the frozen, 4-bit quantized base weight.
* "QLoRA vs ChatGPT", capability 5: the base weight is dequantized on the fly
  in the forward pass; in the backward pass gradients are computed only for the
  LoRA parameters (no gradient for W).
* QLoRA errata page, finding on paper p.4 Section 2: the input gradients exist
  and are kept (activation gradients flow to earlier layers).

Readings: Y = X W'^T + s (X A^T) B^T with s = alpha / r computed in fp32;
W' is the dequantized weight (the bf16 values the format decodes to, not the
original W); no LoRA dropout. All products are fp64 numpy matmuls of the exact
bf16 input values.
"""
from __future__ import annotations

import numpy as np


def lora_scale(alpha: float, r: int) -> np.float32:
    """s = (float) alpha / (float) r, one fp32 division."""
    return np.float32(np.float32(alpha) / np.float32(r))


def linear_fwd(Wd: np.ndarray, X: np.ndarray, A: np.ndarray, B: np.ndarray, s) -> tuple:
    """Y = X W'^T + s (X A^T) B^T.  Shapes: Wd [N,K], X [M,K], A [r,K], B [N,r].

    Returns (Y [M,N], T [M,r]) in fp64, T = X A^T being the saved LoRA input.
    """
    Wd, X, A, B = (np.asarray(t, dtype=np.float64) for t in (Wd, X, A, B))
    s = np.float64(s)
    T = X @ A.T
    Y = X @ Wd.T + s * (T @ B.T)
    return Y, T


def linear_bwd(Wd: np.ndarray, X: np.ndarray, A: np.ndarray, B: np.ndarray, dY: np.ndarray, s) -> tuple:
    """Gradients of the forward map with W frozen.

    dX = dY W' + s (dY B) A
    dA = s (dY B)^T X
    dB = s dY^T (X A^T)
    Returns (dX [M,K], dA [r,K], dB [N,r]) in fp64.
    """
    Wd, X, A, B, dY = (np.asarray(t, dtype=np.float64) for t in (Wd, X, A, B, dY))
    s = np.float64(s)
    U = dY @ B
    dX = dY @ Wd + s * (U @ A)
    dA = s * (U.T @ X)
    dB = s * (dY.T @ (X @ A.T))
    return dX, dA, dB
