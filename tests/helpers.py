"""Shared test helpers: conversions between torch bf16 tensors and the oracle's
numpy representations, error metrics, and the device check for GPU tests."""
from __future__ import annotations

import numpy as np
import torch


def bf16_to_f32_np(t: torch.Tensor) -> np.ndarray:
    """bf16 torch tensor (any device) -> exact fp32 numpy array."""
    return t.detach().float().cpu().numpy()


def bf16_bits_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def rel_fro(got: np.ndarray, ref: np.ndarray) -> float:
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def require_gpu():
    """GPU tests fail (not skip) when the device or the built library is missing."""
    assert torch.cuda.is_available(), "this test needs a CUDA device"
    from bit_nf4_quantized_absmax_b200 import load_library
    load_library()
    return torch.device("cuda:0")


# Tolerance for GEMM outputs and gradients: relative Frobenius error against the
# fp64 oracle (bf16 rounding of the output alone contributes ~1.1e-3 rms).
GEMM_REL_TOL = 2e-3
# Below this many elements the rms of the bf16 output rounding is a noisy
# estimate and can exceed GEMM_REL_TOL by chance; such outputs are checked
# element by element against one bf16 rounding (half an ulp, at most 2^-8
# relative) plus an fp32 accumulation allowance.
SMALL_OUTPUT = 256


def gemm_close(got: np.ndarray, ref: np.ndarray) -> tuple[bool, float]:
    """North-star criterion for GEMM outputs; returns (ok, rel_fro)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    e = rel_fro(got, ref)
    if ref.size >= SMALL_OUTPUT:
        return e < GEMM_REL_TOL, e
    amax = float(np.max(np.abs(ref))) if ref.size else 0.0
    ok = bool(np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * amax + 1e-30))
    return ok, e
