"""Pins for the CPU oracle: checks against facts that do not come from the
oracle itself (library routines it does not call, exact rational arithmetic,
closed forms, brute force on tiny inputs, figures the pages print).

Each test names the plausible oracle mistake it would catch.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special as sp
import torch

import oracle
from oracle import nf4 as onf4
from oracle.fp import bf16_bits_to_f32, f32_to_bf16_bits_rn, fma_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(20261202)


# ----------------------------------------------------------------------------
# exact helpers written for the tests (independent of the oracle's routes)

def frac_round_f32(x: Fraction) -> np.float32:
    """Correct round-to-nearest-even of an exact rational to fp32 by brute force
    over the fp32 neighbours of a first guess."""
    f = np.float32(float(x))
    cands = {f}
    g = f
    for _ in range(2):
        g = np.nextafter(g, np.float32(np.inf)); cands.add(g)
    g = f
    for _ in range(2):
        g = np.nextafter(g, np.float32(-np.inf)); cands.add(g)
    best = sorted(cands, key=lambda c: (abs(Fraction(float(c)) - x),
                                        int(np.array(c, np.float32).view(np.uint32)) & 1))
    return np.float32(best[0])


def frac_argmin_code(v: np.float32, cb: np.ndarray) -> int:
    """Nearest codebook index with exact rational distances; ties -> lower."""
    fv = Fraction(float(v))
    d = [abs(fv - Fraction(float(c))) for c in cb]
    m = min(d)
    return d.index(m)


# ----------------------------------------------------------------------------
# codebook

def test_codebook_invariants():
    """Catches: a missing exact zero, wrong end values, a wrong positive/negative
    split (8 + 0 + 7 uses all 16 patterns), non-monotone ordering."""
    cb = oracle.nf4_codebook()
    assert cb.dtype == np.float32 and cb.shape == (16,)
    assert cb[0] == np.float32(-1.0) and cb[15] == np.float32(1.0) and cb[7] == np.float32(0.0)
    assert np.all(np.diff(cb) > 0)
    assert np.sum(cb < 0) == 7 and np.sum(cb > 0) == 8
    assert len(set(cb.tolist())) == 16


def test_codebook_quantiles_match_scipy_ndtri():
    """The oracle inverts Phi by bisection on erfc; scipy's ndtri is an independent
    routine. Catches a wrong inverse-normal (sign, sqrt 2 factor, bracket)."""
    c64 = onf4.nf4_codebook_f64()
    d = 929.0 / 960.0
    top = sp.ndtri(d)
    pos = np.array([sp.ndtri(0.5 + (d - 0.5) * j / 8) for j in range(1, 9)]) / top
    neg = -np.array([sp.ndtri(0.5 + (d - 0.5) * j / 7) for j in range(1, 8)]) / top
    ref = np.sort(np.concatenate([neg, [0.0], pos]))
    np.testing.assert_allclose(c64, ref, rtol=0, atol=4e-15)


def test_codebook_equal_probability_spacing():
    """Forward check with scipy's ndtr: mapped back through Phi, the codes sit at
    equally spaced probabilities on each side (8 steps above 1/2, 7 below).
    Catches a dropped index, an off-by-one in the split, or a wrong delta."""
    c64 = onf4.nf4_codebook_f64()
    d = 929.0 / 960.0
    top = sp.ndtri(d)
    p = sp.ndtr(c64 * top)
    pos_steps = np.diff(p[7:])
    neg_steps = np.diff(p[:8])
    np.testing.assert_allclose(pos_steps, (d - 0.5) / 8, rtol=1e-12)
    np.testing.assert_allclose(neg_steps, (d - 0.5) / 7, rtol=1e-12)
    assert abs(p[15] - d) < 1e-14 and abs(p[0] - (1 - d)) < 1e-14


def test_codebook_denser_near_zero():
    """NF4 puts more codes where normal weights are dense (near zero): the gaps
    between neighbouring codes grow away from zero on each side."""
    cb = onf4.nf4_codebook_f64()
    gaps_pos = np.diff(cb[7:])
    gaps_neg = np.diff(cb[:8])[::-1]          # from zero outward
    assert np.all(np.diff(gaps_pos) > 0)
    assert np.all(np.diff(gaps_neg) > 0)


def test_codebook_fp32_rounding_is_robust():
    """Every fp64 code value lies far (> 2^-40 relative) from an fp32 rounding
    midpoint, so any correct fp64 construction rounds to the same fp32 bits."""
    c64 = onf4.nf4_codebook_f64()
    for v in c64:
        if v in (0.0, 1.0, -1.0):
            continue
        f = np.float32(v)
        for nb in (np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))):
            mid = (float(f) + float(nb)) / 2
            assert abs(v - mid) > abs(v) * 2.0 ** -40


# ----------------------------------------------------------------------------
# fp helpers

def test_bf16_rounding_matches_torch():
    """Catches a truncating or ties-away bf16 conversion."""
    x = np.concatenate([RNG.standard_normal(20000).astype(np.float32) * 0.05,
                        np.array([0.0, -0.0, 1.0, -1.0, 3.0e-39, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8,
                                  1.0 + 2.0 ** -8 + 2.0 ** -20], dtype=np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(f32_to_bf16_bits_rn(x), ref)
    back = bf16_bits_to_f32(ref)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_fma_single_rounding_exact():
    """fma_f32 against exact rational arithmetic, including the two cases where
    rounding the fp64 sum would land on an fp32 tie and pick the wrong side."""
    a = (RNG.standard_normal(3000) * 4).astype(np.float32)
    b = (RNG.standard_normal(3000) * 1e-3).astype(np.float32)
    c = (RNG.standard_normal(3000) * 0.05).astype(np.float32)
    u = np.float32(1 + 2.0 ** -23)
    adversarial = [
        (u, np.float32((1 - 2.0 ** -23) * 2.0 ** -24), u),      # t on a tie, exact below it
        (u, np.float32(-(1 - 2.0 ** -23) * 2.0 ** -24), u),     # t on a tie, exact above it
        (np.float32(3.0), np.float32(0.0), np.float32(-0.0)),
    ]
    a = np.concatenate([a, [t[0] for t in adversarial]]).astype(np.float32)
    b = np.concatenate([b, [t[1] for t in adversarial]]).astype(np.float32)
    c = np.concatenate([c, [t[2] for t in adversarial]]).astype(np.float32)
    got = fma_f32(a, b, c)
    for i in range(a.size):
        x = Fraction(float(a[i])) * Fraction(float(b[i])) + Fraction(float(c[i]))
        assert got[i] == frac_round_f32(x), (i, a[i], b[i], c[i])
    # the adversarial cases really are ones a plain double rounding gets wrong
    naive = (a[-3:-1].astype(np.float64) * b[-3:-1] + c[-3:-1]).astype(np.float32)
    assert np.all(naive != got[-3:-1])


# ----------------------------------------------------------------------------
# first-level quantization

def test_nearest_code_brute_force_rational():
    """Exact rational distances on random v and on v placed at, just below and
    just above every decision midpoint. Catches ties going to the upper index,
    a distance taken in fp32, or a shifted index."""
    cb = oracle.nf4_codebook()
    vs = list(RNG.uniform(-1, 1, 3000).astype(np.float32))
    for i in range(15):
        mid = (float(cb[i]) + float(cb[i + 1])) / 2
        f = np.float32(mid)
        vs += [f, np.nextafter(f, np.float32(1)), np.nextafter(f, np.float32(-1))]
    vs += [np.float32(-1.0), np.float32(1.0), np.float32(0.0), np.float32(-0.0), np.float32(1e-30)]
    vs = np.array(vs, dtype=np.float32)
    got = onf4.nearest_code(vs, cb)
    for v, g in zip(vs, got):
        assert g == frac_argmin_code(v, cb), v


def test_exact_tie_goes_to_lower_index():
    """Where a midpoint of two neighbouring codes is itself an fp32 number, the
    midpoint must map to the lower index."""
    cb = oracle.nf4_codebook()
    ties = 0
    for i in range(15):
        mid = Fraction(float(cb[i])) / 2 + Fraction(float(cb[i + 1])) / 2
        f = np.float32(float(mid))
        if Fraction(float(f)) == mid:
            ties += 1
            assert onf4.nearest_code(np.array([f]), cb)[0] == i
    # the zero/neighbour midpoints are half of an fp32 value, always representable
    assert ties >= 2


def _rand_bf16(shape, std=0.02, seed=0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16).float().numpy()


def test_quantize_brute_force_small():
    """Block absmax, the fp32 division and the nearest code, all redone with
    exact rationals on a tiny weight. Catches a reciprocal-multiply, a block that
    spans the wrong elements, or a wrong block size."""
    W = _rand_bf16((3, 128), seed=1)
    W[1, 64:128] = 0.0                       # an all-zero block
    cb = oracle.nf4_codebook()
    codes, absmax = onf4.quantize_nf4(W, cb)
    blocks = W.reshape(-1, 64)
    for b in range(blocks.shape[0]):
        m = max(abs(Fraction(float(x))) for x in blocks[b])
        assert Fraction(float(absmax[b])) == m
        for j in range(64):
            if m == 0:
                want = 7
            else:
                v = frac_round_f32(Fraction(float(blocks[b, j])) / m)
                want = frac_argmin_code(v, cb)
            assert codes[b * 64 + j] == want


def test_block_extreme_maps_to_end_code():
    W = _rand_bf16((4, 256), seed=2)
    codes, absmax = onf4.quantize_nf4(W, oracle.nf4_codebook())
    blocks = W.reshape(-1, 64)
    cblk = codes.reshape(-1, 64)
    for b in range(blocks.shape[0]):
        j = int(np.argmax(np.abs(blocks[b])))
        assert cblk[b, j] == (15 if blocks[b, j] > 0 else 0)


def test_pack_order_low_nibble_first():
    """The stored byte i holds element 2i in its low nibble (the layout the
    library documents)."""
    codes = np.array([1, 2, 15, 0, 7, 8], dtype=np.uint8)
    assert onf4.pack_codes(codes).tolist() == [0x21, 0x0F, 0x87]
    assert onf4.unpack_codes(onf4.pack_codes(codes)).tolist() == codes.tolist()


def test_requantize_dequantized_is_idempotent():
    """quantize(dequant(quantize(W))) reproduces the codes: bf16 and DQ errors
    (<= 2^-8 relative) are far below half the smallest code gap (~0.04)."""
    for dist_seed in (3, 4):
        W = _rand_bf16((64, 512), seed=dist_seed)
        qw = oracle.quantize_nf4_dq(W)
        Wd = bf16_bits_to_f32(oracle.dequantize_nf4_dq(qw))
        qw2 = oracle.quantize_nf4_dq(Wd)
        assert np.array_equal(qw.packed, qw2.packed)


# ----------------------------------------------------------------------------
# double quantization

def test_dq_mean_is_exact_sum():
    """The mean uses the exact sum of the constants: a wide dynamic range where a
    left-to-right fp64 sum is inexact still gives fp64(S)/n correctly."""
    m = np.array([2.0 ** 40, 2.0 ** -40, -0.0 + 1.0, 2.0 ** -40, 3.0], dtype=np.float32)
    mu = onf4.dq_mean(m)
    S = sum(Fraction(float(x)) for x in m)
    assert mu == np.float32(float(S) / 5.0)
    naive = np.float32(np.float64(np.sum(m.astype(np.float64))) / 5.0)
    assert mu == naive  # here both agree; the next case shows order dependence
    m2 = np.array([1.0, 2.0 ** -53, 2.0 ** -53, -0.0], dtype=np.float32)
    S2 = sum(Fraction(float(x)) for x in m2)
    assert Fraction(float(math.fsum(m2.astype(np.float64).tolist()))) == S2


def test_dq_closed_forms():
    """All-equal constants: mu equals them, every group has s_g = 0 and the
    decoded constants are exactly the originals. A two-valued group maps its
    extremes to -127 / +127."""
    m = np.full(700, 0.0390625, dtype=np.float32)
    q, sc, mu = onf4.double_quantize(m)
    assert mu == np.float32(0.0390625) and np.all(q == 0) and np.all(sc == 0)
    assert np.array_equal(onf4.dequant_constants(q, sc, mu), m)
    m = np.array([1.0, 3.0] * 128, dtype=np.float32)
    q, sc, mu = onf4.double_quantize(m)
    assert mu == np.float32(2.0) and sc[0] == np.float32(1.0 / 127.0)
    assert q.tolist() == [-127, 127] * 128


def test_dq_rint_ties_to_even_and_bound():
    """Codes are rint (ties to even) of an fp32 quotient, and each decoded
    constant is within half a step (+1 ulp) of the original."""
    # a group whose scale is exactly 1/127 * 127 = 1 -> quotients 0.5, 1.5, 2.5
    # offsets sum to zero so the mean is exactly 200
    m = np.array([127.0, 0.5, 1.5, 2.5, -127.0, -4.5], dtype=np.float32) + np.float32(200.0)
    q, sc, mu = onf4.double_quantize(m)
    assert mu == np.float32(200.0) and sc[0] == np.float32(1.0)
    assert q.tolist() == [127, 0, 2, 2, -127, -4]
    W = _rand_bf16((256, 1024), seed=5)
    codes, absmax = onf4.quantize_nf4(W, oracle.nf4_codebook())
    q, sc, mu = onf4.double_quantize(absmax)
    mp = onf4.dequant_constants(q, sc, mu)
    grp = np.arange(absmax.size) // 256
    err = np.abs(mp.astype(np.float64) - absmax.astype(np.float64))
    ulp = np.spacing(np.abs(mp)).astype(np.float64)
    assert np.all(err <= sc[grp].astype(np.float64) / 2 + 2 * ulp)
    assert q.min() >= -127 and q.max() <= 127


def _dq_codes_exact(c: list, mu: np.float32) -> tuple:
    """Int8 codes and scale of one group by exact rational arithmetic, written
    from the definition: c_b = fp32(m_b - mu), s = max |c_b|, scale =
    fp32(s / 127), q_b = clamp(round-half-even(fp32(c_b / scale)), -127, 127)."""
    cc = [frac_round_f32(Fraction(float(m)) - Fraction(float(mu))) for m in c]
    s = max(abs(Fraction(float(x))) for x in cc)
    scale = frac_round_f32(s / 127)
    if scale == 0:
        return [0] * len(cc), scale
    out = []
    for x in cc:
        quo = Fraction(float(frac_round_f32(Fraction(float(x)) / Fraction(float(scale)))))
        fl = math.floor(quo)
        d = quo - fl
        k = fl + 1 if (d > Fraction(1, 2) or (d == Fraction(1, 2) and fl % 2 == 1)) else fl
        out.append(max(-127, min(127, int(k))))
    return out, scale


def test_dq_quotient_exact_rationals():
    """The int8 code of each constant is round-half-even of the fp32-rounded
    quotient c_b / scale ("QLoRA vs ChatGPT", capability 3: the first-level
    constants are quantized to 8 bit with scales of their own).

    Checked against exact rationals on 10^4 random groups (a sample of their
    constants by Fraction, all of them through an fp64 quotient rounded once to
    fp32, which is the correctly rounded fp32 quotient because 53 >= 2*24 + 2),
    and on constructed constants whose quotient lies within a few fp32 ulps of
    k + 1/2, where rounding the quotient to fp32 first decides the code: there
    a reciprocal multiply, or rounding the unrounded quotient, gives other codes."""
    rng = np.random.default_rng(777)
    ngrp = 10_000
    m = np.abs(_rand_bf16((ngrp, 256), std=0.02, seed=3)).astype(np.float32).reshape(-1)
    m = np.maximum(m, np.float32(1e-4))
    mu = np.float32(0.0123)
    q, sc, mu_out = onf4.double_quantize(m, mean=mu)
    assert mu_out == mu and sc.shape == (ngrp,)
    # every constant: fp64 quotient of the two fp32 values, one rounding to fp32, rint (ties to even)
    c = (m - mu).astype(np.float32)
    grp = np.arange(m.size) // 256
    ref = np.rint(np.float32(c.astype(np.float64) / sc[grp].astype(np.float64)))
    assert np.array_equal(q.astype(np.int64), np.clip(ref, -127, 127).astype(np.int64))
    # a random sample of groups by exact rationals
    for g in rng.choice(ngrp, 12, replace=False):
        want, scale = _dq_codes_exact(m[256 * g:256 * (g + 1)].tolist(), mu)
        assert sc[g] == scale
        assert q[256 * g:256 * (g + 1)].tolist() == want

    # constructed near-ties: scale fixed by one constant, the others near (k + 1/2) * scale
    cases_recip, cases_unrounded, checked = 0, 0, 0
    for trial in range(40):
        s = np.float32(rng.uniform(0.01, 0.2))
        scale = frac_round_f32(Fraction(float(s)) / 127)
        group = [s]
        for k in rng.integers(-126, 126, size=24):
            target = np.float32((k + 0.5) * float(scale))
            x = target
            for step in range(-3, 4):
                y = x
                for _ in range(abs(step)):
                    y = np.nextafter(y, np.float32(np.inf if step > 0 else -np.inf))
                if abs(float(y)) <= float(s):
                    group.append(np.float32(y))
        group = np.array(group, dtype=np.float32)
        q, sc, _ = onf4.double_quantize(group, mean=np.float32(0.0))
        want, scale_x = _dq_codes_exact(group.tolist(), np.float32(0.0))
        assert sc[0] == scale_x and q.tolist() == want
        checked += group.size
        r = np.float32(np.float32(1.0) / sc[0])
        recip = np.clip(np.rint(np.float32(group * r)), -127, 127).astype(int)
        unrounded = np.clip(np.rint(group.astype(np.float64) / np.float64(sc[0])), -127, 127).astype(int)
        cases_recip += int(np.sum(recip != np.array(want)))
        cases_unrounded += int(np.sum(unrounded != np.array(want)))
    assert checked > 5000
    # the construction has teeth: both plausible wrong quotient steps disagree somewhere
    assert cases_recip > 0 and cases_unrounded > 0


def test_dq_groups_of_256_and_ragged_tail():
    """Group boundaries at multiples of 256 constants; the last group shorter."""
    m = np.concatenate([np.full(256, 1.0), np.full(256, 2.0), np.array([3.0, 5.0])]).astype(np.float32)
    q, sc, mu = onf4.double_quantize(m)
    assert sc.shape == (3,)
    S = Fraction(256) + Fraction(512) + Fraction(8)
    assert mu == np.float32(float(S) / 514.0)
    # group 2 holds only the two tail constants
    c = np.array([3.0, 5.0], np.float32) - mu
    assert sc[2] == np.float32(np.max(np.abs(c)) / np.float32(127))


# ----------------------------------------------------------------------------
# storage overhead against the pages' printed figures

def test_storage_overhead_matches_pages():
    g = json.load(open(os.path.join(GOLDEN, "storage_claims.json")))
    K = 4096
    dq = onf4.storage_bytes(4096, K, True)
    single = onf4.storage_bytes(4096, K, False)
    # closed form: 4 + 8/64 + 32/(64*256) bit vs 4 + 32/64
    assert abs(dq["bits_per_param"] - (4 + 8 / 64 + 32 / (64 * 256)) - 32 / (4096 * K)) < 1e-12
    assert abs(single["bits_per_param"] - 4.5) < 1e-12
    saving = single["bits_per_param"] - dq["bits_per_param"]
    assert abs(saving - g["dq_saving_bits_per_param"]["value"]) <= g["dq_saving_bits_per_param"]["abs_tol"]
    comp = 16.0 / dq["bits_per_param"]
    assert abs(comp / g["compression_vs_16bit"]["value"] - 1) <= g["compression_vs_16bit"]["rel_tol"]
    # the oracle's arrays have exactly the sizes the format claims
    W = _rand_bf16((8, 8192), seed=6)
    qw = oracle.quantize_nf4_dq(W)
    sb = onf4.storage_bytes(8, 8192, True)
    assert qw.packed.nbytes == sb["packed"] and qw.absmax_q.nbytes == sb["absmax_q"]
    assert qw.dq_scale.nbytes == sb["dq_scale"]
    # Llama-65B linear weights in NF4+DQ fit the 48 GB GPU and the 41 GB table row
    shapes = g["llama65b_linear_shapes"]["value"]
    total = g["llama65b_linear_shapes"]["layers"] * sum(onf4.storage_bytes(n, k)["total"] for n, k in shapes)
    assert 30e9 < total < g["model_size_65b_4bit_GB"]["value"] * 1e9 < g["gpu_memory_65b_finetune_GB"]["value"] * 1e9


# ----------------------------------------------------------------------------
# dequantization

def test_dequant_exhaustive_codes_and_qvalues():
    """All 16 codes x 255 int8 constant codes for fixed (scale, mean), against
    exact rationals: fma with one rounding, product rounded to fp32, then bf16."""
    cb = oracle.nf4_codebook()
    sc = np.float32(0.000123456)
    mu = np.float32(0.0431)
    q = np.arange(-127, 128, dtype=np.int8)
    mp = onf4.dequant_constants(q, np.array([sc]), mu) if q.size <= 256 else None
    for qi, mpi in zip(q.tolist(), mp):
        want = frac_round_f32(Fraction(qi) * Fraction(float(sc)) + Fraction(float(mu)))
        assert mpi == want
    codes = np.tile(np.arange(16, dtype=np.uint8), 4)  # one 64-block per q value
    for qi in (-127, -1, 0, 1, 64, 127):
        qw = onf4.QuantizedNF4(onf4.pack_codes(codes), np.array([qi], np.int8), np.array([sc]), mu, 1, 64,
                               np.zeros(1, np.float32))
        got = onf4.dequantize_nf4_dq(qw).reshape(-1)
        mpi = frac_round_f32(Fraction(qi) * Fraction(float(sc)) + Fraction(float(mu)))
        for j in range(64):
            prod = frac_round_f32(Fraction(float(cb[codes[j]])) * Fraction(float(mpi)))
            ref = torch.tensor([float(prod)], dtype=torch.float32).to(torch.bfloat16).view(torch.int16)
            assert got[j] == (int(ref.item()) & 0xFFFF)


# ----------------------------------------------------------------------------
# linear forward / backward

def _tiny_linear(M=3, N=5, K=64, r=2, seed=7):
    g = torch.Generator().manual_seed(seed)
    f = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16).double().numpy()
    return f(N, K) * 0.02, f(M, K), f(r, K) * 0.1, f(N, r) * 0.1, f(M, N)


def test_fwd_bwd_match_triple_loops():
    """Pure-Python loops for every product (catches a transposed operand or a
    missing scale)."""
    Wd, X, A, B, dY = _tiny_linear()
    s = float(oracle.lora_scale(16, 2))
    M, K = X.shape; N = Wd.shape[0]; r = A.shape[0]
    Y, T = oracle.linear_fwd(Wd, X, A, B, s)
    dX, dA, dB = oracle.linear_bwd(Wd, X, A, B, dY, s)
    for m in range(M):
        Tm = [sum(X[m, k] * A[j, k] for k in range(K)) for j in range(r)]
        for j in range(r):
            assert abs(T[m, j] - Tm[j]) < 1e-12
        for n in range(N):
            y = sum(X[m, k] * Wd[n, k] for k in range(K)) + s * sum(Tm[j] * B[n, j] for j in range(r))
            assert abs(Y[m, n] - y) < 1e-12
        for k in range(K):
            U = [sum(dY[m, n] * B[n, j] for n in range(N)) for j in range(r)]
            v = sum(dY[m, n] * Wd[n, k] for n in range(N)) + s * sum(U[j] * A[j, k] for j in range(r))
            assert abs(dX[m, k] - v) < 1e-12
    for j in range(r):
        for k in range(K):
            v = s * sum(sum(dY[m, n] * B[n, j] for n in range(N)) * X[m, k] for m in range(M))
            assert abs(dA[j, k] - v) < 1e-12
    for n in range(N):
        for j in range(r):
            v = s * sum(dY[m, n] * sum(X[m, k] * A[j, k] for k in range(K)) for m in range(M))
            assert abs(dB[n, j] - v) < 1e-12


def test_adjoint_identities():
    """<dY, Y> = <dX, X> (Y linear in X); <dA, A> = <dB, B> = s <dY, X A^T B^T>."""
    Wd, X, A, B, dY = _tiny_linear(M=7, N=9, K=128, r=4, seed=8)
    s = 0.25
    Y, _ = oracle.linear_fwd(Wd, X, A, B, s)
    dX, dA, dB = oracle.linear_bwd(Wd, X, A, B, dY, s)
    lora = s * (X @ A.T) @ B.T
    assert abs(np.sum(dY * Y) - np.sum(dX * X)) < 1e-10
    assert abs(np.sum(dA * A) - np.sum(dY * lora)) < 1e-10
    assert abs(np.sum(dB * B) - np.sum(dY * lora)) < 1e-10


def test_finite_differences():
    """Central differences of L = <dY, Y>: exact up to rounding for a bilinear map.
    Catches a wrong sign or a gradient taken for the wrong operand."""
    Wd, X, A, B, dY = _tiny_linear(M=4, N=6, K=64, r=3, seed=9)
    s = 0.5
    L = lambda X_, A_, B_: float(np.sum(dY * oracle.linear_fwd(Wd, X_, A_, B_, s)[0]))
    dX, dA, dB = oracle.linear_bwd(Wd, X, A, B, dY, s)
    h = 1e-3
    for (arr, grad, which) in ((X, dX, 0), (A, dA, 1), (B, dB, 2)):
        for _ in range(6):
            idx = tuple(RNG.integers(0, n) for n in arr.shape)
            args_p = [X.copy(), A.copy(), B.copy()]
            args_m = [X.copy(), A.copy(), B.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            fd = (L(*args_p) - L(*args_m)) / (2 * h)
            assert abs(fd - grad[idx]) < 1e-9 * max(1.0, abs(grad[idx]))


def test_lora_scale_fp32():
    assert oracle.lora_scale(16, 64) == np.float32(0.25)
    assert oracle.lora_scale(16, 16) == np.float32(1.0)
    assert oracle.lora_scale(1, 3) == np.float32(1.0) / np.float32(3.0)
