"""Oracle for the NF4 data type, block-wise absmax quantization, double
quantization of the absmax constants and block-wise dequantization.

Test infrastructure only (see the package docstring). Plain numpy/Python; every
rounding that decides a stored bit pattern is exact.

Passages followed:
* NF4 values: "Guanaco", section "Technical Innovations" (a 4-bit type for
  normally distributed weights, denser near zero); the QLoRA errata page,
  finding on paper p.5 Section 3 (the data type has a discrete zero point and
  uses all 2^k values of a k-bit type); "QLoRA vs ChatGPT", capability 1
  (NF4 optimized for normally distributed weights).
* Block-wise absmax quantization: "QLoRA vs ChatGPT", capability 1
  (block-wise quantization with absmax scaling of the base weights).
* Double quantization: "Guanaco", section "Core Architecture & Training"
  (quantizing the quantization constants saves about 0.4 bit per parameter);
  "QLoRA vs ChatGPT", capability 3 (the first-level constants are quantized to
  8 bit and stored with their own scales, a nested hierarchy).
* Dequantization: "QLoRA vs ChatGPT", capability 5 (weights are dequantized
  on the fly, block by block, in the forward pass).
* Single-level storage (no double quantization): the QLoRA errata page,
  findings on the paper's p.8 Table 4, which compares NFloat4 with and without
  DQ; "QLoRA vs ChatGPT", capability 3, which contrasts the nested scheme with
  keeping the constants as full-precision metadata. The first-level constants
  m_b are stored as fp32 and used directly as the block scale.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from fractions import Fraction

import numpy as np

from .fp import f32_to_bf16_bits_rn, fma_f32

BLOCK = 64        # weights per first-level absmax block
DQ_BLOCK = 256    # first-level constants per second-level (8-bit) block

# Reading: the pages print neither the NF4 construction nor its offset. The
# codebook is built from normal quantiles at equally spaced probabilities
# between 1/2 and delta, with delta the mean of the half-bin offsets of a
# 15-bin and a 16-bin equal-probability split: delta = 1 - (1/30 + 1/32)/2.
DELTA = Fraction(1) - (Fraction(1, 30) + Fraction(1, 32)) / 2   # = 929/960
N_POS = 8   # positive codes (indices 8..15)
N_NEG = 7   # negative codes (indices 0..6); index 7 is the exact zero


def _phi(x: float) -> float:
    """Standard normal CDF, 0.5*erfc(-x/sqrt 2) (host libm erfc)."""
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def _phi_inv(p: float) -> float:
    """Inverse standard normal CDF for p in (1/2, 1) by bisection on _phi.

    Bisection runs until the bracket is two adjacent doubles; the endpoint with
    the smaller |_phi(x) - p| is returned.
    """
    assert 0.5 < p < 1.0
    lo, hi = 0.0, 40.0
    while True:
        mid = 0.5 * (lo + hi)
        if mid == lo or mid == hi:
            break
        if _phi(mid) < p:
            lo = mid
        else:
            hi = mid
    return lo if abs(_phi(lo) - p) <= abs(_phi(hi) - p) else hi


def nf4_codebook_f64() -> np.ndarray:
    """The 16 NF4 values in fp64, ascending, before rounding to fp32.

    Positive side: Phi^-1(1/2 + (delta - 1/2) j / 8), j = 1..8.
    Negative side: -Phi^-1(1/2 + (delta - 1/2) j / 7), j = 1..7.
    Plus an exact 0, then everything divided by Phi^-1(delta) so that the end
    values are exactly -1 and +1. 7 negatives + 0 + 8 positives use all 16
    four-bit patterns and keep a discrete zero.
    """
    half = Fraction(1, 2)
    pos = [_phi_inv(float(half + (DELTA - half) * j / N_POS)) for j in range(1, N_POS + 1)]
    neg = [-_phi_inv(float(half + (DELTA - half) * j / N_NEG)) for j in range(1, N_NEG + 1)]
    top = _phi_inv(float(DELTA))
    vals = sorted(neg + [0.0] + pos)
    return np.array([v / top for v in vals], dtype=np.float64)


def nf4_codebook() -> np.ndarray:
    """The NF4 codebook as fp32[16] (round-to-nearest of the fp64 values)."""
    return nf4_codebook_f64().astype(np.float32)


def fp4_codebook() -> np.ndarray:
    """The FP4 comparison codebook as fp32[16], ascending.

    Reading (the QLoRA errata page's findings on the paper's p.8 Table 4 compare
    NFloat4 with Float4; the pages give no format): the 4-bit float with one sign
    bit, two exponent bits e and one mantissa bit f, exponent bias 1, with
    subnormals at e = 0: value = f / 2 for e = 0, (1 + f / 2) * 2^(e - 1)
    otherwise. Divided by its largest magnitude so the range is [-1, 1], like
    NF4. Its +0 and -0 are one value, kept once: the 15 distinct values fill
    indices 0..14 and index 15 repeats the largest value, which the nearest code
    (ties to the lower index) never selects.
    """
    mags = set()
    for e in range(4):
        for f in range(2):
            mags.add(Fraction(f, 2) if e == 0 else (1 + Fraction(f, 2)) * Fraction(2) ** (e - 1))
    top = max(mags)
    vals = sorted({s * m / top for m in mags for s in (1, -1)})
    assert len(vals) == 15
    vals.append(vals[-1])
    out = np.empty(16, dtype=np.float32)
    for i, v in enumerate(vals):
        out[i] = _fraction_to_f32(v)
    return out


def _fraction_to_f32(x: Fraction) -> np.float32:
    """Round an exact rational to the nearest fp32 (ties to even): the two fp32
    neighbours of the fp64 value bracket it, and the nearer one wins."""
    f = np.float32(float(x))
    best = f
    for g in (np.nextafter(f, np.float32(-np.inf)), np.nextafter(f, np.float32(np.inf))):
        dg, db = abs(Fraction(float(g)) - x), abs(Fraction(float(best)) - x)
        if dg < db or (dg == db and int(np.array(g).view(np.uint32)) % 2 == 0):
            best = g
    return np.float32(best)


def nearest_code(v: np.ndarray, codebook: np.ndarray) -> np.ndarray:
    """argmin_i |v - c_i| for fp32 v in [-1, 1]; ties go to the lower index.

    Distances are taken in fp64. Near any decision midpoint |v| > 2^-30, and the
    difference of two fp32 numbers whose exponents lie within 29 of each other
    is exact in fp64, so every comparison that can be close is exact; np.argmin
    returns the first minimum, i.e. the lower index on a tie.
    """
    cb = np.asarray(codebook, dtype=np.float32).astype(np.float64)
    d = np.abs(np.asarray(v, dtype=np.float32).astype(np.float64)[..., None] - cb)
    return np.argmin(d, axis=-1).astype(np.uint8)


def quantize_nf4(W: np.ndarray, codebook: np.ndarray, chunk_blocks: int = 1 << 14):
    """First-level quantization of a bf16-valued weight (given as fp32).

    W: [N, K] with K % 64 == 0; blocks are 64 consecutive elements in row-major
    order, so a block never crosses a row. Per block b: m_b = max |w| (exact in
    fp32). If m_b == 0 all codes are 7 (the exact zero). Otherwise
    v = fp32(w / m_b) (IEEE division) and code = nearest_code(v).
    Returns (codes uint8 [N*K], absmax fp32 [N*K/64]).
    """
    W = np.ascontiguousarray(W, dtype=np.float32)
    if W.ndim != 2 or W.shape[1] % BLOCK:
        raise ValueError("W must be [N, K] with K a multiple of 64")
    if not np.all(np.isfinite(W)):
        raise ValueError("oracle inputs must be finite")
    blocks = W.reshape(-1, BLOCK)
    nblk = blocks.shape[0]
    absmax = np.max(np.abs(blocks), axis=1) if nblk else np.zeros(0, np.float32)
    codes = np.full(blocks.shape, 7, dtype=np.uint8)
    for s in range(0, nblk, chunk_blocks):
        e = min(nblk, s + chunk_blocks)
        m = absmax[s:e]
        nz = m > 0
        if not np.any(nz):
            continue
        v = blocks[s:e][nz] / m[nz][:, None]          # fp32 / fp32, correctly rounded
        c = codes[s:e]
        c[nz] = nearest_code(v, codebook)
    return codes.reshape(-1), absmax.astype(np.float32)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte: element 2i in the low nibble, 2i+1 in the high nibble."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1, 2)
    return (c[:, 0] | (c[:, 1] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p & 0xF
    out[1::2] = p >> 4
    return out


def dq_mean(absmax: np.ndarray) -> np.float32:
    """mu = fp32(fp64(S) / nblk) with S the exact sum of the absmax constants.

    math.fsum returns the correctly rounded sum, so fp64(S) does not depend on
    the summation order; the division is an fp64 division, then one rounding
    to fp32.
    """
    n = absmax.size
    if n == 0:
        return np.float32(0.0)
    S = math.fsum(np.asarray(absmax, dtype=np.float64).tolist())
    return np.float32(np.float64(S) / np.float64(n))


def double_quantize(absmax: np.ndarray, mean=None):
    """Second-level quantization of the fp32 absmax constants to int8.

    mu = dq_mean(absmax); c_b = fp32(m_b - mu). Per group of 256 consecutive
    constants (the last group may be shorter): s_g = max |c_b|,
    dq_scale_g = fp32(s_g / 127), q_b = clamp(rint_even(fp32(c_b / dq_scale_g)),
    -127, 127). A group with s_g == 0 gets dq_scale_g = 0 and q_b = 0.
    `mean`, when given, is the mean of a larger set of constants that `absmax`
    is a group-aligned part of (a row shard of the weight), used in place of
    dq_mean(absmax).
    Returns (q int8 [nblk], dq_scale fp32 [ngrp], mu fp32).
    """
    m = np.asarray(absmax, dtype=np.float32)
    n = m.size
    mu = dq_mean(m) if mean is None else np.float32(mean)
    c = (m - mu).astype(np.float32)
    ngrp = (n + DQ_BLOCK - 1) // DQ_BLOCK
    cp = np.zeros(ngrp * DQ_BLOCK, dtype=np.float32)
    cp[:n] = c
    g = cp.reshape(ngrp, DQ_BLOCK)
    s = np.max(np.abs(g), axis=1) if ngrp else np.zeros(0, np.float32)
    scale = (s / np.float32(127.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = (g / scale[:, None]).astype(np.float32)
    qf = np.rint(ratio)
    qf = np.where(s[:, None] > 0, qf, 0.0)
    qf = np.clip(qf, -127, 127)
    q = qf.astype(np.int8).reshape(-1)[:n]
    return q, scale.astype(np.float32), np.float32(mu)


@dataclass
class QuantizedNF4:
    """NF4 + double-quant storage of one [rows, cols] weight."""
    packed: np.ndarray     # uint8 [rows*cols/2]
    absmax_q: np.ndarray   # int8 [nblk]
    dq_scale: np.ndarray   # fp32 [ngrp]
    mean: np.float32       # fp32
    rows: int
    cols: int
    absmax: np.ndarray     # fp32 [nblk], first-level constants (not stored by the format)


def quantize_nf4_dq(W: np.ndarray, codebook: np.ndarray | None = None) -> QuantizedNF4:
    cb = nf4_codebook() if codebook is None else codebook
    codes, absmax = quantize_nf4(W, cb)
    q, scale, mu = double_quantize(absmax)
    return QuantizedNF4(pack_codes(codes), q, scale, mu, W.shape[0], W.shape[1], absmax)


def dequant_constants(q: np.ndarray, dq_scale: np.ndarray, mean) -> np.ndarray:
    """m'_b = fmaf((float) q_b, dq_scale_g, mu): one rounding to fp32."""
    q = np.asarray(q, dtype=np.int8)
    grp = np.arange(q.size) // DQ_BLOCK
    return fma_f32(q.astype(np.float32), np.asarray(dq_scale, np.float32)[grp], np.float32(mean))


def dequantize_nf4_dq(qw: QuantizedNF4, codebook: np.ndarray | None = None) -> np.ndarray:
    """w' = bf16_rn(fp32(c[code] * m'_b)); returns bf16 bit patterns [rows, cols]."""
    cb = (nf4_codebook() if codebook is None else codebook).astype(np.float32)
    codes = unpack_codes(qw.packed).reshape(-1, BLOCK)
    mprime = dequant_constants(qw.absmax_q, qw.dq_scale, qw.mean)
    prod = (cb[codes] * mprime[:, None]).astype(np.float32)
    return f32_to_bf16_bits_rn(prod).reshape(qw.rows, qw.cols)


@dataclass
class QuantizedNF4Single:
    """Single-level NF4 storage of one [rows, cols] weight: codes and fp32 m_b."""
    packed: np.ndarray     # uint8 [rows*cols/2]
    absmax: np.ndarray     # fp32 [nblk]
    rows: int
    cols: int


def quantize_nf4_single(W: np.ndarray, codebook: np.ndarray | None = None) -> QuantizedNF4Single:
    """Level-1 quantization alone: the codes of quantize_nf4 and its exact m_b."""
    cb = nf4_codebook() if codebook is None else codebook
    codes, absmax = quantize_nf4(W, cb)
    return QuantizedNF4Single(pack_codes(codes), absmax, W.shape[0], W.shape[1])


def dequantize_nf4_single(qw: QuantizedNF4Single, codebook: np.ndarray | None = None) -> np.ndarray:
    """w' = bf16_rn(fp32(c[code] * m_b)) with the stored m_b; bf16 bit patterns [rows, cols]."""
    cb = (nf4_codebook() if codebook is None else codebook).astype(np.float32)
    codes = unpack_codes(qw.packed).reshape(-1, BLOCK)
    m = np.asarray(qw.absmax, dtype=np.float32)
    prod = (cb[codes] * m[:, None]).astype(np.float32)
    return f32_to_bf16_bits_rn(prod).reshape(qw.rows, qw.cols)


def storage_bytes(rows: int, cols: int, double_quant: bool = True) -> dict:
    """Bytes the stored format takes for one [rows, cols] weight."""
    numel = rows * cols
    nblk = numel // BLOCK
    ngrp = (nblk + DQ_BLOCK - 1) // DQ_BLOCK
    if double_quant:
        d = {"packed": numel // 2, "absmax_q": nblk, "dq_scale": 4 * ngrp, "mean": 4}
    else:
        d = {"packed": numel // 2, "absmax": 4 * nblk}
    d["total"] = sum(d.values())
    d["bits_per_param"] = 8.0 * d["total"] / numel
    return d
