"""GPU parity of qlora_merge_lora (weighted adapters merged into the NF4 base),
bit-exact against the oracle, through the C ABI."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_absmax_b200 import binding as b
from bit_nf4_quantized_absmax_b200 import synthetic as syn
from tests.helpers import bf16_bits_np, bf16_to_f32_np, require_gpu

pytestmark = pytest.mark.gpu


def _case(N, K, ranks, seed):
    W = syn.normal_bf16((N, K), 0.02, seed, "test", 100)
    ads = []
    for i, r in enumerate(ranks):
        A = syn.normal_bf16((r, K), 0.02, seed, "test", 101 + 2 * i)
        B = syn.normal_bf16((N, r), 0.02, seed, "test", 102 + 2 * i)
        ads.append((A, B))
    return W, ads


def _oracle_merge(W, ads, alphas, weights, rows=None):
    qw = oracle.quantize_nf4_dq(bf16_to_f32_np(W))
    Wd = oracle.dequantize_nf4_dq(qw)
    spec = []
    for (A, B), al, wt in zip(ads, alphas, weights):
        Bn = bf16_to_f32_np(B)
        spec.append((bf16_to_f32_np(A), Bn if rows is None else Bn[rows], A.shape[0], al, wt))
    return oracle.merge_lora(Wd if rows is None else Wd[rows], spec)


@pytest.mark.parametrize("N,K,ranks,alphas,weights", [
    (256, 512, (16,), (16.0,), (1.0,)),
    (100, 320, (8, 24), (16.0, 8.0), (0.7, -0.3)),
    (64, 1088, (64, 8, 128), (16.0, 32.0, 64.0), (0.5, 1.0, 0.25)),
    (17, 64, (256,), (16.0,), (2.0,)),
])
def test_merge_bit_exact(N, K, ranks, alphas, weights):
    dev = require_gpu()
    W, ads = _case(N, K, ranks, 7)
    q = b.qlora_quantize_nf4_dq(W.to(dev))
    gpu_ads = [(A.to(dev), B.to(dev), al, wt) for (A, B), al, wt in zip(ads, alphas, weights)]
    out = b.qlora_merge_lora(q, gpu_ads)
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    assert np.array_equal(bf16_bits_np(out), _oracle_merge(W, ads, alphas, weights))


def test_merge_without_adapters_is_the_dequant():
    dev = require_gpu()
    W, _ = _case(96, 256, (), 3)
    q = b.qlora_quantize_nf4_dq(W.to(dev))
    out = b.qlora_merge_lora(q, [])
    ref = b.qlora_dequantize_nf4_dq(q)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_merged_weight_requantizes_like_the_oracle():
    dev = require_gpu()
    W, ads = _case(128, 512, (32,), 11)
    q = b.qlora_quantize_nf4_dq(W.to(dev))
    merged = b.qlora_merge_lora(q, [(ads[0][0].to(dev), ads[0][1].to(dev), 16.0, 1.0)])
    q2 = b.qlora_quantize_nf4_dq(merged)
    torch.cuda.synchronize()
    ref_bits = _oracle_merge(W, ads, (16.0,), (1.0,))
    ref_q = oracle.quantize_nf4_dq(oracle.bf16_bits_to_f32(ref_bits))
    assert np.array_equal(q2.packed.cpu().numpy(), ref_q.packed)
    assert np.array_equal(q2.absmax_q.cpu().numpy(), ref_q.absmax_q)
    assert np.array_equal(q2.dq_scale.cpu().numpy().view(np.uint32), ref_q.dq_scale.view(np.uint32))


def test_merge_llama7b_mlp_sampled_rows():
    dev = require_gpu()
    N, K, r = 11008, 4096, 64
    W, ads = _case(N, K, (r,), 0)
    q = b.qlora_quantize_nf4_dq(W.to(dev))
    out = b.qlora_merge_lora(q, [(ads[0][0].to(dev), ads[0][1].to(dev), 16.0, 1.0)])
    torch.cuda.synchronize()
    rows = np.concatenate([[0, N - 1], np.random.default_rng(0).choice(N, 30, replace=False)])
    assert np.array_equal(bf16_bits_np(out)[rows], _oracle_merge(W, ads, (16.0,), (1.0,), rows=rows))
