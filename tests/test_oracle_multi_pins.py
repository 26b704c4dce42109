"""Pins of the oracle's several-adapters forward ("QLoRA vs ChatGPT",
capability 6: adapters composed with weights), CPU only: it equals the sum of
single-adapter forwards (each checked with a pure-Python triple loop on a tiny
shape), it equals the forward of the unrounded merged weight, one adapter of
weight 1 is the ordinary forward, and a weight of zero drops an adapter."""
from __future__ import annotations

import numpy as np

import oracle
from oracle.merge import merge_scale


def _case(M=3, N=5, K=64, ranks=(2, 3), seed=11):
    rng = np.random.default_rng(seed)
    Wd = rng.standard_normal((N, K))
    X = rng.standard_normal((M, K))
    ads = []
    for i, r in enumerate(ranks):
        ads.append((rng.standard_normal((r, K)), rng.standard_normal((N, r)), float(8 * (i + 1)), 0.5 + i))
    return Wd, X, ads


def test_multi_equals_triple_loop_sum():
    Wd, X, ads = _case()
    Y = oracle.linear_fwd_multi(Wd, X, ads)
    M, K = X.shape
    N = Wd.shape[0]
    for m in range(M):
        for n in range(N):
            ref = sum(X[m, k] * Wd[n, k] for k in range(K))
            for A, B, alpha, w in ads:
                c = float(merge_scale(alpha, A.shape[0], w))
                t = [sum(X[m, k] * A[j, k] for k in range(K)) for j in range(A.shape[0])]
                ref += c * sum(t[j] * B[n, j] for j in range(A.shape[0]))
            assert abs(Y[m, n] - ref) <= 1e-11 * (1 + abs(ref))


def test_multi_equals_merged_weight_forward():
    Wd, X, ads = _case(M=4, N=7, K=128, ranks=(8, 16, 8), seed=12)
    merged = Wd.copy()
    for A, B, alpha, w in ads:
        merged += np.float64(merge_scale(alpha, A.shape[0], w)) * (B @ A)
    assert np.allclose(oracle.linear_fwd_multi(Wd, X, ads), X @ merged.T, rtol=1e-12, atol=1e-10)


def test_one_adapter_weight_one_is_the_forward_and_zero_weight_drops():
    Wd, X, ads = _case(ranks=(4,), seed=13)
    A, B, alpha, _ = ads[0]
    Y1 = oracle.linear_fwd_multi(Wd, X, [(A, B, alpha, 1.0)])
    Yf, _ = oracle.linear_fwd(Wd, X, A, B, oracle.lora_scale(alpha, A.shape[0]))
    assert np.allclose(Y1, Yf, rtol=1e-13, atol=1e-12)
    Y0 = oracle.linear_fwd_multi(Wd, X, [(A, B, alpha, 0.0)])
    assert np.allclose(Y0, X @ Wd.T, rtol=1e-13, atol=1e-12)
