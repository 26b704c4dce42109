"""Pins of the oracle's FP4 codebook (the Float4 type that the QLoRA errata
page's findings on the paper's p.8 Table 4 compare with NFloat4) and of the
library's host table for it. CPU only.

Reading (the pages give no FP4 format): 1 sign, 2 exponent and 1 mantissa bit,
magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6} divided by 6, zero kept once, index 15
repeating +1 (never selected: ties go to the lower index)."""
from __future__ import annotations

from fractions import Fraction

import numpy as np

import oracle
from oracle import nf4 as onf4
from tests.test_oracle_pins import frac_argmin_code, frac_round_f32

# the textbook 1-2-1 minifloat magnitudes over 6, written out as rationals
FP4_RATIONALS = [Fraction(-6, 6), Fraction(-4, 6), Fraction(-3, 6), Fraction(-2, 6), Fraction(-3, 12),
                 Fraction(-1, 6), Fraction(-1, 12), Fraction(0), Fraction(1, 12), Fraction(1, 6), Fraction(3, 12),
                 Fraction(2, 6), Fraction(3, 6), Fraction(4, 6), Fraction(6, 6), Fraction(6, 6)]


def test_fp4_codebook_values():
    cb = oracle.fp4_codebook()
    want = np.array([frac_round_f32(x) for x in FP4_RATIONALS], dtype=np.float32)
    assert np.array_equal(cb.view(np.uint32), want.view(np.uint32))
    assert cb[0] == -1.0 and cb[7] == 0.0 and cb[14] == 1.0 and cb[15] == 1.0
    assert np.all(np.diff(cb[:15]) > 0) and np.count_nonzero(cb == 0.0) == 1
    # the value set is closed under negation and uses exactly 15 distinct values
    assert sorted(set((-cb).tolist())) == sorted(set(cb.tolist())) and len(set(cb.tolist())) == 15


def test_fp4_nearest_code_brute_force_and_unused_index():
    cb = oracle.fp4_codebook()
    rng = np.random.default_rng(41)
    v = np.concatenate([rng.uniform(-1, 1, 4000).astype(np.float32),
                        np.array([1.0, -1.0, 0.0, 1 / 24, -1 / 24, 5 / 6, 7 / 12], np.float32)])
    got = onf4.nearest_code(v, cb)
    want = np.array([frac_argmin_code(x, cb) for x in v])
    assert np.array_equal(got, want)
    assert 15 not in got.tolist() and got[v == 1.0].tolist() == [14]
    # exact midpoints tie to the lower index; one fp32 step above goes up
    for i in range(14):
        mid = (Fraction(float(cb[i])) + Fraction(float(cb[i + 1]))) / 2
        f = np.float32(float(mid))
        if Fraction(float(f)) == mid:
            assert onf4.nearest_code(np.array([f]), cb)[0] == i
            up = np.nextafter(f, np.float32(2))
            assert onf4.nearest_code(np.array([up]), cb)[0] == i + 1


def test_fp4_quantize_small_against_rationals():
    rng = np.random.default_rng(43)
    W = (rng.standard_normal((3, 128)) * 0.05).astype(np.float32)
    W = np.array([[float(np.float32(x)) for x in row] for row in W], dtype=np.float32)
    W[1, :64] = 0.0
    cb = oracle.fp4_codebook()
    codes, absmax = onf4.quantize_nf4(W, cb)
    blocks = W.reshape(-1, 64)
    for b, blk in enumerate(blocks):
        m = max(abs(Fraction(float(x))) for x in blk)
        assert Fraction(float(absmax[b])) == m
        for k, x in enumerate(blk):
            want = 7 if m == 0 else frac_argmin_code(frac_round_f32(Fraction(float(x)) / m), cb)
            assert codes[b * 64 + k] == want


def test_library_fp4_codebook_bits():
    from bit_nf4_quantized_absmax_b200 import binding as b
    lib_cb = b.qlora_codebook(b.DTYPE_FP4).numpy()
    assert np.array_equal(lib_cb.view(np.uint32), oracle.fp4_codebook().view(np.uint32))
    assert np.array_equal(b.qlora_codebook(b.DTYPE_NF4).numpy().view(np.uint32),
                          oracle.nf4_codebook().view(np.uint32))
