"""Pins of the single-level NF4 oracle (oracle.quantize_nf4_single /
dequantize_nf4_single) against facts that do not come from its own formula:
exact rational rounding, the codebook's exact end points, the double-quantized
format in the case where its constants are lossless, and the storage sizes the
pages compare."""
from __future__ import annotations

from fractions import Fraction

import numpy as np

import oracle
from oracle.fp import bf16_bits_to_f32, f32_to_bf16_bits_rn


def _bf16(x):
    return bf16_bits_to_f32(f32_to_bf16_bits_rn(np.asarray(x, dtype=np.float32)))


def _round_rational(x: Fraction, p: int) -> Fraction:
    """x rounded to p significant bits, nearest, ties to even (normal range)."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    scale = Fraction(2) ** (p - 1 - e)
    y = a * scale
    n = y.numerator // y.denominator
    rem = y - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * Fraction(n) / scale


def test_dequant_equals_exact_two_step_rounding():
    """w' = bf16(fp32(c * m)), each rounding done on exact rationals."""
    rng = np.random.default_rng(11)
    W = _bf16(rng.standard_normal((3, 128)) * 0.02)
    qw = oracle.quantize_nf4_single(W)
    got = bf16_bits_to_f32(oracle.dequantize_nf4_single(qw)).reshape(-1)
    cb = oracle.nf4_codebook()
    codes = oracle.unpack_codes(qw.packed)
    for i, code in enumerate(codes):
        m = Fraction(float(qw.absmax[i // 64]))
        exact = Fraction(float(cb[code])) * m
        want = _round_rational(_round_rational(exact, 24), 8)
        assert Fraction(float(got[i])) == want, i


def test_block_maximum_decodes_to_itself():
    """codebook[0] = -1 and codebook[15] = +1 exactly and m_b is a bf16 value, so
    the element of largest magnitude in every block comes back unchanged."""
    rng = np.random.default_rng(12)
    W = _bf16(rng.standard_t(4, (16, 256)) * 0.02)
    qw = oracle.quantize_nf4_single(W)
    Wd = bf16_bits_to_f32(oracle.dequantize_nf4_single(qw))
    blocks, dblocks = W.reshape(-1, 64), Wd.reshape(-1, 64)
    for b in range(blocks.shape[0]):
        j = int(np.argmax(np.abs(blocks[b])))
        assert dblocks[b, j] == blocks[b, j]
        assert qw.absmax[b] == abs(blocks[b, j])


def test_matches_double_quantized_format_when_its_constants_are_lossless():
    """If every block has the same absmax m, the mean is m, every centred constant
    is 0 and the double-quantized block constant fmaf(0, 0, m) is m exactly: both
    formats then decode to the same bits."""
    rng = np.random.default_rng(13)
    W = _bf16(rng.uniform(-0.5, 0.5, (8, 512)) * 0.02)
    W.reshape(-1, 64)[:, 5] = np.float32(0.015625)  # a power of two above every other |w|
    single = oracle.dequantize_nf4_single(oracle.quantize_nf4_single(W))
    dq = oracle.quantize_nf4_dq(W)
    assert np.all(dq.absmax_q == 0) and np.all(dq.dq_scale == 0) and dq.mean == np.float32(0.015625)
    assert np.array_equal(single, oracle.dequantize_nf4_dq(dq))


def test_zero_block_decodes_to_zero():
    W = np.zeros((2, 128), np.float32)
    W[1, 70] = 0.25
    qw = oracle.quantize_nf4_single(W)
    Wd = bf16_bits_to_f32(oracle.dequantize_nf4_single(qw))
    assert qw.absmax[0] == 0 and qw.absmax[1] == 0
    assert np.all(Wd[0] == 0) and np.all(Wd[1, :64] == 0) and Wd[1, 70] == np.float32(0.25)


def test_double_quantization_saves_about_0_4_bit_per_parameter():
    """The pages: quantizing the constants saves about 0.4 bit per parameter
    against keeping them in 32 bit (one per 64 weights: 0.5 bit)."""
    single = oracle.storage_bytes(8192, 8192, double_quant=False)["bits_per_param"]
    dq = oracle.storage_bytes(8192, 8192, double_quant=True)["bits_per_param"]
    assert single == 4.5
    assert abs((single - dq) - 0.373) < 0.001
    assert round(single - dq, 1) == 0.4
