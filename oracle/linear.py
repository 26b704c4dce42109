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


def linear_fwd_multi(Wd: np.ndarray, X: np.ndarray, adapters) -> np.ndarray:
    """Several adapters applied at once without merging them ("QLoRA vs
    ChatGPT", capability 6: adapters trained on one quantized base are composed
    with weights): Y = X W'^T + sum_a c_a (X A_a^T) B_a^T in fp64, with
    c_a = fp32(w_a * fp32(alpha_a / r_a)), the composition scale of the merge.

    adapters: sequence of (A_a [r_a, K], B_a [N, r_a], alpha_a, w_a).
    Reading: the pages name the composition, not its arithmetic; the scale of an
    adapter is the one its merge into the weights uses. Returns Y [M, N].
    """
    Wd, X = np.asarray(Wd, dtype=np.float64), np.asarray(X, dtype=np.float64)
    Y = X @ Wd.T
    for A, B, alpha, w in adapters:
        A, B = np.asarray(A, dtype=np.float64), np.asarray(B, dtype=np.float64)
        s = np.float32(np.float32(alpha) / np.float32(A.shape[0]))
        c = np.float64(np.float32(np.float32(w) * s))
        Y = Y + c * ((X @ A.T) @ B.T)
    return Y

