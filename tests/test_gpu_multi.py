"""Several LoRA adapters at inference without merging ("QLoRA vs ChatGPT",
capability 6), through the C ABI: the pack call lays the adapters side by side
bit for bit, and the forward equals the fp64 oracle Y = X W'^T + sum_a c_a
(X A_a^T) B_a^T within the GEMM tolerance on the decode kernels (M <= 16, both
kinds) and the tensor-core path (M > 16)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle.merge import merge_scale
from bit_nf4_quantized_absmax_b200 import binding as b
from bit_nf4_quantized_absmax_b200 import synthetic as syn
from tests.helpers import bf16_to_f32_np, gemm_close, require_gpu

pytestmark = pytest.mark.gpu


def _adapters(N, K, ranks, weights, seed, dev):
    ads = []
    for i, (r, w) in enumerate(zip(ranks, weights)):
        A = syn.normal_bf16((r, K), 0.02, seed, "test", 700 + 3 * i).to(dev)
        B = syn.normal_bf16((N, r), 0.02, seed, "test", 701 + 3 * i).to(dev)
        ads.append((A, B, float(4 * (i + 2)), w))
    return ads


def _check(N, K, M, ranks, weights, seed=5):
    dev = require_gpu()
    W = syn.normal_bf16((N, K), 0.02, seed, "test", 690).to(dev)
    X = syn.normal_bf16((M, K), 1.0, seed, "test", 691).to(dev)
    q = b.qlora_quantize_nf4_dq(W)
    ads = _adapters(N, K, ranks, weights, seed, dev)
    A_cat, B_cat, cs = b.qlora_pack_adapters(ads, N, K)
    Y = b.qlora_linear_fwd_multi(q, X, A_cat, B_cat, cs)
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    # the packed operands are the adapters side by side, the scales the merge's
    assert torch.equal(A_cat, torch.cat([a[0] for a in ads], 0))
    assert torch.equal(B_cat, torch.cat([a[1] for a in ads], 1))
    want = np.concatenate([np.full(a[0].shape[0], merge_scale(a[2], a[0].shape[0], a[3]), np.float32) for a in ads])
    assert np.array_equal(cs.cpu().numpy().view(np.uint32), want.view(np.uint32))
    Wd = oracle.bf16_bits_to_f32(oracle.dequantize_nf4_dq(oracle.quantize_nf4_dq(bf16_to_f32_np(W.cpu()))))
    f64 = lambda t: bf16_to_f32_np(t).astype(np.float64)  # noqa: E731
    Yr = oracle.linear_fwd_multi(Wd.astype(np.float64), f64(X),
                                 [(f64(A), f64(B), alpha, w) for A, B, alpha, w in ads])
    ok, e = gemm_close(bf16_to_f32_np(Y), Yr)
    assert ok, e
    return q, X, ads, Y


@pytest.mark.parametrize("M", [1, 5, 16])
def test_multi_decode(M):
    _check(512, 1024, M, ranks=(8, 16, 64), weights=(1.0, 0.5, -0.25))


def test_multi_decode_llama7b_shape():
    _check(4096, 4096, 1, ranks=(64, 64), weights=(0.7, 0.3))


@pytest.mark.parametrize("M", [64, 300])
def test_multi_tensor_core(M):
    _check(512, 1024, M, ranks=(16, 24, 8), weights=(1.0, -0.5, 2.0))


def test_one_adapter_matches_the_forward():
    q, X, ads, Y = _check(1024, 768, 9, ranks=(32,), weights=(1.0,))
    A, B, alpha, _ = ads[0]
    Y1, _ = b.qlora_linear_fwd(q, X, A, B, alpha)
    torch.cuda.synchronize()
    d = (Y.float() - Y1.float()).abs().max().item()
    assert d <= 2.0 ** -7 * Y1.float().abs().max().item()  # same sum, scale applied at a different point


def test_pack_errors():
    dev = require_gpu()
    A = torch.zeros(8, 128, dtype=torch.bfloat16, device=dev)
    B = torch.zeros(64, 8, dtype=torch.bfloat16, device=dev)
    with pytest.raises(b.QloraError):
        b.qlora_pack_adapters([(A, B, 8.0, 1.0)] * 9, 64, 128)   # more than 8 adapters
    big = torch.zeros(136, 128, dtype=torch.bfloat16, device=dev)
    bigB = torch.zeros(64, 136, dtype=torch.bfloat16, device=dev)
    with pytest.raises(b.QloraError):
        b.qlora_pack_adapters([(big, bigB, 8.0, 1.0), (big, bigB, 8.0, 1.0)], 64, 128)  # sum r > 256
