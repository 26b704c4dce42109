"""Oracle: merging LoRA adapters into the dequantized base weight (test
infrastructure only; see the package docstring).

Follows "QLoRA vs ChatGPT" (unfragile.ai compare page), capability blurb 6:
several adapters trained on one quantized base can be composed with weights
(w1 * adapter1 + w2 * adapter2) and merged into the base weights to give a
standalone checkpoint. The pages give no arithmetic for the merge; the reading
taken here (and by the library) is:

    y = W'[n, k]                                   (the bf16 dequantized base, exact in fp64)
    for each adapter a, in the given order:
        P = sum over j = 0 .. r_a - 1, in order, of B_a[n, j] * A_a[j, k]      (fp64)
        c = fp32(w_a * s_a),  s_a = fp32(alpha_a / r_a)
        y = fp64(y + fp64(c * P))
    W_merged[n, k] = bf16_rn(y)                    (one rounding from fp64)

Every product B_a[n, j] * A_a[j, k] of two bf16 values is exact in fp64 (at most
16 significant bits), so each step of the sum rounds once, in a fixed order; the
result is therefore a fixed function of the inputs that any fp64 implementation
following the same order reproduces bit for bit.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def f64_to_bf16_bits_rn(y: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns, round to nearest, ties to even, in one step,
    on the integer bit pattern (vectorized). ``f64_to_bf16_bits_rn_exact`` is the
    same rounding done on exact rationals, element by element (slow; used to
    pin this one)."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    if not np.all(np.isfinite(y)):
        raise ValueError("oracle inputs must be finite")
    u = y.view(np.uint64)
    sign = ((u >> np.uint64(48)) & np.uint64(0x8000)).astype(np.uint64)
    e = ((u >> np.uint64(52)) & np.uint64(0x7FF)).astype(np.int64)
    m = (u & np.uint64((1 << 52) - 1)).astype(np.uint64)
    # significand with the hidden bit (doubles below 2^-1022 have no hidden bit;
    # they are far below the bf16 range and round to zero below)
    sig = np.where(e > 0, m | np.uint64(1 << 52), m)
    E = np.where(e > 0, e - 1023, -1022)          # value = sig * 2^(E - 52)
    # bf16 keeps 8 significant bits for E >= -126; below, the grid is 2^-133
    shift = np.where(E >= -126, 45, 45 + (-126 - E)).astype(np.int64)  # bits dropped from sig
    big = shift >= 64
    sh = np.minimum(shift, 63).astype(np.uint64)
    keep = np.where(big, np.uint64(0), sig >> sh)
    rem = np.where(big, sig, sig & ((np.uint64(1) << sh) - np.uint64(1)))
    half = np.where(big, np.uint64(0), np.uint64(1) << (sh - np.uint64(1)))
    up = np.where(big, False, (rem > half) | ((rem == half) & ((keep & np.uint64(1)) == 1)))
    keep = keep + up.astype(np.uint64)
    # assemble: normal range keeps 8 bits incl. the hidden one; exponent field E + 127
    normal = E >= -126
    expf = np.where(normal, E + 127, 0).astype(np.int64)
    # a carry out of the 8-bit significand moves to the next binade
    carry = normal & (keep >= np.uint64(256))
    keep = np.where(carry, keep >> np.uint64(1), keep)
    expf = np.where(carry, expf + 1, expf)
    # subnormal results that round up to 2^-126 become the smallest normal
    sub_up = (~normal) & (keep >= np.uint64(128))
    expf = np.where(sub_up, 1, expf)
    mant = np.where(normal | sub_up, keep & np.uint64(0x7F), keep)
    bits = np.where(expf >= 255, np.uint64(0x7F80), (expf.astype(np.uint64) << np.uint64(7)) | mant)
    bits = np.where(y == 0, np.uint64(0), bits)
    return (bits | sign).astype(np.uint16)


def f64_to_bf16_bits_rn_exact(y: np.ndarray) -> np.ndarray:
    """The same rounding on exact rationals, one element at a time."""
    y = np.asarray(y, dtype=np.float64)
    if not np.all(np.isfinite(y)):
        raise ValueError("oracle inputs must be finite")
    out = np.empty(y.shape, dtype=np.uint16)
    flat = y.ravel()
    res = out.ravel()
    for i, v in enumerate(flat):
        res[i] = _f64_to_bf16_one(float(v))
    return out


def _f64_to_bf16_one(v: float) -> int:
    sign = 0x8000 if (v < 0 or (v == 0 and np.signbit(v))) else 0
    x = Fraction(abs(v))
    if x == 0:
        return sign
    # exponent E with 2^E <= x < 2^(E+1)
    E = x.numerator.bit_length() - x.denominator.bit_length()
    if Fraction(2) ** E > x:
        E -= 1
    E = max(E, -126)
    q = Fraction(2) ** (E - 7)  # grid spacing
    k_floor = x // q
    rem = x - k_floor * q
    if rem * 2 > q or (rem * 2 == q and k_floor % 2 == 1):
        k = k_floor + 1
    else:
        k = k_floor
    val = k * q
    if val >= Fraction(2) ** 128:
        return sign | 0x7F80
    # encode val = k * 2^(E-7)
    if k < 128:  # subnormal (only possible with E == -126)
        return sign | int(k)
    if k == 256:  # rounded up to the next binade
        k = 128
        E += 1
    exp_field = E + 127
    return sign | (exp_field << 7) | (int(k) - 128)


def merge_scale(alpha: float, r: int, weight: float) -> np.float32:
    """c = fp32(w * s) with s = fp32(alpha / r): two fp32 roundings."""
    s = np.float32(np.float32(alpha) / np.float32(r))
    return np.float32(np.float32(weight) * s)


def merge_lora(Wd_bits: np.ndarray, adapters) -> np.ndarray:
    """Merged bf16 bit patterns [N, K] from the bf16 base W' (bit patterns) and
    a list of adapters (A [r, K] bf16 values as fp32, B [N, r] likewise, r,
    alpha, weight), in the order given (reading above)."""
    Wd_bits = np.asarray(Wd_bits, dtype=np.uint16)
    y = (Wd_bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    for (A, B, r, alpha, weight) in adapters:
        A = np.asarray(A, dtype=np.float32).astype(np.float64)
        B = np.asarray(B, dtype=np.float32).astype(np.float64)
        assert A.shape[0] == r and B.shape[1] == r
        P = np.zeros_like(y)
        for j in range(r):
            P = P + np.outer(B[:, j], A[j, :])  # exact products, one rounding per step
        c = np.float64(merge_scale(alpha, r, weight))
        y = y + c * P
    return f64_to_bf16_bits_rn(y)
