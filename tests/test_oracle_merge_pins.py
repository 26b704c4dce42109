"""Pins of the adapter-merge oracle (oracle/merge.py) against facts that do not
come from the oracle itself: exact rational arithmetic, torch's own fp32->bf16
rounding, hand-derived cases, and the order the reading fixes."""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import torch

from oracle import merge as om
from oracle.fp import bf16_bits_to_f32, f32_to_bf16_bits_rn


def _bits(x):
    return np.asarray(x, dtype=np.uint16)


def test_f64_to_bf16_matches_exact_rationals():
    rng = np.random.default_rng(1)
    b = rng.integers(0, 0x7F7F, 4000).astype(np.uint16)
    lo = bf16_bits_to_f32(b).astype(np.float64)
    hi = bf16_bits_to_f32(b + 1).astype(np.float64)
    mids = (lo + hi) / 2  # exact bf16 midpoints (ties)
    edge = np.array([0.0, -0.0, 1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 2.0 ** -126, 2.0 ** -133, 2.0 ** -134,
                     3 * 2.0 ** -134, 2.0 ** -126 * (1 - 2.0 ** -9), 3.3895313892515355e38, 3.39e38, 1e-300, 5e-324])
    x = np.concatenate([edge, mids, -mids, rng.standard_normal(5000) * 0.02,
                        np.exp(rng.uniform(-120, 88, 3000)) * rng.choice([-1.0, 1.0], 3000)])
    assert np.array_equal(om.f64_to_bf16_bits_rn(x), om.f64_to_bf16_bits_rn_exact(x))


def test_f64_to_bf16_agrees_with_torch_on_fp32_values():
    """For values that are already fp32, one rounding from fp64 equals torch's fp32->bf16."""
    rng = np.random.default_rng(2)
    f = (rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))).astype(np.float32)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(om.f64_to_bf16_bits_rn(f.astype(np.float64)), ref)


def test_f64_to_bf16_hand_cases():
    assert om.f64_to_bf16_bits_rn(np.array([1 + 2.0 ** -8]))[0] == 0x3F80      # tie -> even (1.0)
    assert om.f64_to_bf16_bits_rn(np.array([1 + 3 * 2.0 ** -8]))[0] == 0x3F82  # tie -> even (1 + 2^-6)
    assert om.f64_to_bf16_bits_rn(np.array([1 + 2.0 ** -8 + 2.0 ** -40]))[0] == 0x3F81  # just above the tie
    assert om.f64_to_bf16_bits_rn(np.array([-0.0]))[0] == 0x8000
    assert om.f64_to_bf16_bits_rn(np.array([2.0 ** -134]))[0] == 0x0000        # half the smallest subnormal -> 0
    assert om.f64_to_bf16_bits_rn(np.array([3 * 2.0 ** -134]))[0] == 0x0002    # 1.5 units -> 2 (even)
    assert om.f64_to_bf16_bits_rn(np.array([3.4e38]))[0] == 0x7F80             # above the top midpoint


def _rand_bf16(rng, shape, std):
    return bf16_bits_to_f32(f32_to_bf16_bits_rn((rng.standard_normal(shape) * std).astype(np.float32)))


def test_no_adapter_or_zero_weight_returns_the_base():
    rng = np.random.default_rng(3)
    Wd = f32_to_bf16_bits_rn((rng.standard_normal((16, 64)) * 0.02).astype(np.float32))
    A, B = _rand_bf16(rng, (8, 64), 0.02), _rand_bf16(rng, (16, 8), 0.02)
    assert np.array_equal(om.merge_lora(Wd, []), Wd)
    assert np.array_equal(om.merge_lora(Wd, [(A, B, 8, 16.0, 0.0)]), Wd)


def test_exact_case_equals_rational_arithmetic():
    """Small powers of two make every fp64 step exact: the merge is then the
    exact rational W' + c B A rounded once to bf16."""
    rng = np.random.default_rng(4)
    N, K, r = 8, 16, 8
    Wd = f32_to_bf16_bits_rn(np.ldexp(rng.integers(-8, 8, (N, K)).astype(np.float32), -6))
    A = np.ldexp(rng.integers(-4, 5, (r, K)).astype(np.float32), -3)
    B = np.ldexp(rng.integers(-4, 5, (N, r)).astype(np.float32), -5)
    alpha, w = 16.0, 0.75
    got = om.merge_lora(Wd, [(A, B, r, alpha, w)])
    c = Fraction(float(np.float32(np.float32(w) * np.float32(np.float32(alpha) / np.float32(r)))))
    W0 = bf16_bits_to_f32(Wd)
    for n in range(N):
        for k in range(K):
            exact = Fraction(float(W0[n, k])) + c * sum(Fraction(float(B[n, j])) * Fraction(float(A[j, k]))
                                                       for j in range(r))
            assert got[n, k] == om.f64_to_bf16_bits_rn_exact(np.array([float(exact)]))[0]


def test_sum_runs_in_adapter_index_order_in_fp64():
    """Products 2^60, 1, -2^60 in that order: fp64 sums to 0 (the 1 is absorbed);
    an exact sum would give 1. The reading fixes the sequential fp64 sum."""
    K, r = 1, 8
    A = np.zeros((r, K), np.float32)
    B = np.zeros((1, r), np.float32)
    A[:3, 0] = [2.0 ** 30, 1.0, 2.0 ** 30]
    B[0, :3] = [2.0 ** 30, 1.0, -(2.0 ** 30)]
    Wd = f32_to_bf16_bits_rn(np.array([[0.5]], np.float32))
    got = om.merge_lora(Wd, [(A, B, r, float(r), 1.0)])  # c = 1
    assert got[0, 0] == 0x3F00  # 0.5 + 0
    B[0, :3] = [1.0, 2.0 ** 30, -(2.0 ** 30)]  # 1 first: 1 + 2^60 - 2^60 = 0 as well in fp64
    A[:3, 0] = [1.0, 2.0 ** 30, 2.0 ** 30]
    assert om.merge_lora(Wd, [(A, B, r, float(r), 1.0)])[0, 0] == 0x3F00
    B[0, :3] = [2.0 ** 30, -(2.0 ** 30), 1.0]  # cancellation first: 0 + 1 = 1
    A[:3, 0] = [2.0 ** 30, 2.0 ** 30, 1.0]
    assert om.merge_lora(Wd, [(A, B, r, float(r), 1.0)])[0, 0] == 0x3FC0  # 1.5


def test_adapters_apply_in_the_given_order():
    """y = (W' + c1 P1) + c2 P2 in fp64: with W' = 1, c1 P1 = 2^60 and
    c2 P2 = -2^60 the 1 is absorbed by the first step, so the result is 0; an
    exact sum would give 1."""
    r = 8
    A1 = np.zeros((r, 1), np.float32); B1 = np.zeros((1, r), np.float32)
    A2 = np.zeros((r, 1), np.float32); B2 = np.zeros((1, r), np.float32)
    A1[0, 0], B1[0, 0] = 2.0 ** 30, 2.0 ** 30
    A2[0, 0], B2[0, 0] = 2.0 ** 30, -(2.0 ** 30)
    Wd = f32_to_bf16_bits_rn(np.array([[1.0]], np.float32))
    got = om.merge_lora(Wd, [(A1, B1, r, float(r), 1.0), (A2, B2, r, float(r), 1.0)])
    assert got[0, 0] == 0x0000


def test_merge_is_close_to_the_real_sum():
    rng = np.random.default_rng(5)
    N, K, r = 32, 128, 16
    Wd = f32_to_bf16_bits_rn((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    A, B = _rand_bf16(rng, (r, K), 0.02), _rand_bf16(rng, (N, r), 0.02)
    got = bf16_bits_to_f32(om.merge_lora(Wd, [(A, B, r, 32.0, 0.5)])).astype(np.float64)
    ref = bf16_bits_to_f32(Wd).astype(np.float64) + float(om.merge_scale(32.0, r, 0.5)) * (
        B.astype(np.float64) @ A.astype(np.float64))
    # one bf16 rounding: at most half an ulp (2^-8 relative) away
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-30)
