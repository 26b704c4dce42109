"""Exact floating-point helpers for the oracle (test infrastructure only).

numpy gives correctly rounded fp32 +, -, *, / and fp64 arithmetic, but no
fused multiply-add and no bf16 type. The two helpers below supply them exactly:

* ``f32_to_bf16_bits_rn``: IEEE round-to-nearest-even from fp32 to bf16, done on
  the integer bit pattern.
* ``fma_f32``: a*b + c with a single rounding to fp32, for fp32 a, b, c. The
  product of two fp32 values is exact in fp64; the fp64 sum and its exact error
  term (Knuth's TwoSum) then decide the one fp32 rounding.
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> the same values as fp32 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def f32_to_bf16_bits_rn(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest, ties to even (finite inputs)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if not np.all(np.isfinite(x)):
        raise ValueError("oracle inputs must be finite")
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def fma_f32(a, b, c) -> np.ndarray:
    """fp32(a*b + c) with one rounding; a, b, c are fp32 arrays (broadcast).

    p = a*b is exact in fp64 (24+24 significand bits). t = fl64(p + c) and
    e = (p + c) - t exactly (TwoSum), so the exact sum is x = t + e.
    Let lo <= t <= hi be the fp32 neighbours of t and mid their midpoint (an
    fp64 number). Since t is the fp64 rounding of x, x and t lie on the same
    side of mid unless t == mid; in that case the sign of e decides, and e == 0
    is a true tie resolved to the even neighbour.
    """
    a64 = np.asarray(a, dtype=np.float32).astype(np.float64)
    b64 = np.asarray(b, dtype=np.float32).astype(np.float64)
    c64 = np.asarray(c, dtype=np.float32).astype(np.float64)
    p = a64 * b64
    t = p + c64
    bb = t - p
    e = (p - (t - bb)) + (c64 - bb)

    r = t.astype(np.float32)  # RN-even of t: correct unless t is an fp32 midpoint
    r64 = r.astype(np.float64)
    # fp32 neighbours bracketing t
    lo = np.where(r64 <= t, r, np.nextafter(r, np.float32(-np.inf)))
    hi = np.where(r64 >= t, r, np.nextafter(r, np.float32(np.inf)))
    mid = (lo.astype(np.float64) + hi.astype(np.float64)) * 0.5
    on_mid = (lo != hi) & (t == mid) & (e != 0)
    r = np.where(on_mid & (e > 0), hi, r)
    r = np.where(on_mid & (e < 0), lo, r)
    return np.asarray(r, dtype=np.float32)
