"""GPU parity of single-level NF4 storage (fp32 block constants, no double
quantization) against the CPU oracle, through the C ABI: codes, constants and
dequantized weights bit for bit; the linear layer within the GEMM tolerance;
the adapter merge bit for bit."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_absmax_b200 import binding as b
from bit_nf4_quantized_absmax_b200 import synthetic as syn
from tests.helpers import bf16_bits_np, bf16_to_f32_np, gemm_close, require_gpu
from tests.test_gpu_quant import _ratio_tensor

pytestmark = pytest.mark.gpu


def _gpu_single(W_cpu: torch.Tensor):
    dev = require_gpu()
    W = W_cpu.to(dev).contiguous()
    qs = b.qlora_quantize_nf4(W)
    qd = b.qlora_quantize_nf4_dq(W)
    Wd = b.qlora_dequantize_nf4(qs)
    Wd2 = b.qlora_dequantize_nf4_dq(qs)  # the older name takes either kind
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    assert torch.equal(qs.packed, qd.packed)  # level 1 does not depend on level 2
    assert torch.equal(Wd.view(torch.int16), Wd2.view(torch.int16))
    return qs, Wd


def _assert_bit_exact(W_cpu, qs, Wd):
    ref = oracle.quantize_nf4_single(bf16_to_f32_np(W_cpu))
    assert np.array_equal(qs.absmax.cpu().numpy().view(np.uint32), ref.absmax.view(np.uint32))
    got = qs.packed.cpu().numpy()
    if not np.array_equal(got, ref.packed):
        bad = np.nonzero(got != ref.packed)[0]
        raise AssertionError(f"{bad.size} packed bytes differ, first at {bad[:8]}")
    assert np.array_equal(bf16_bits_np(Wd), oracle.dequantize_nf4_single(ref))


@pytest.mark.parametrize("shape", [(1024, 1024), (1, 64), (3, 192), (257, 320), (33, 64 * 300)])
def test_single_quantize_dequant_bit_exact(shape):
    W = syn.normal_bf16(shape, 0.02, 0, "test", shape[0] * 11 + shape[1])
    qs, Wd = _gpu_single(W)
    _assert_bit_exact(W, qs, Wd)


def test_single_edge_blocks():
    """All-zero blocks, signed zeros, huge and subnormal magnitudes."""
    W = syn.normal_bf16((24, 64 * 40), 0.02, 0, "test", 131).float()
    W[0, :64] = 0.0
    W[1, :] = 0.0
    W[2, 64:128] = -0.0
    W[5, :64] *= 2.0 ** 100
    W[6, :64] *= 2.0 ** -120
    W[7, :64] = torch.tensor([2.0 ** -133] * 64)
    Wb = W.to(torch.bfloat16)
    qs, Wd = _gpu_single(Wb)
    _assert_bit_exact(Wb, qs, Wd)


def test_single_every_significand_pair():
    W = _ratio_tensor(seed=9)
    qs, Wd = _gpu_single(W)
    _assert_bit_exact(W, qs, Wd)


def test_single_llama7b_full_size():
    """11008x4096: every constant compared; codes and dequantized values on 66
    rows (single-level rows are independent, so the oracle runs row by row)."""
    shape = (11008, 4096)
    W = syn.normal_bf16(shape, 0.02, 0, "llama7b", 16 * syn.LLAMA7B_SHAPES.index(shape))
    qs, Wd = _gpu_single(W)
    Wf = bf16_to_f32_np(W)
    assert np.array_equal(qs.absmax.cpu().numpy(), np.max(np.abs(Wf.reshape(-1, 64)), axis=1))
    rng = np.random.default_rng(2)
    rows = np.concatenate([[0, shape[0] - 1], np.sort(rng.choice(shape[0], 64, replace=False))])
    packed = qs.packed.cpu().numpy().reshape(shape[0], -1)
    wd = bf16_bits_np(Wd)
    ref = oracle.quantize_nf4_single(Wf[rows])
    assert np.array_equal(packed[rows].reshape(-1), ref.packed)
    assert np.array_equal(wd[rows], oracle.dequantize_nf4_single(ref))


@pytest.mark.parametrize("M,r", [(1, 64), (9, 16), (16, 24), (300, 32)])
def test_single_linear_parity(M, r):
    """Decode (M <= 16) and tensor-core (M = 300) forward, and the backward,
    with single-level storage; the oracle uses its own single-level W'."""
    dev = require_gpu()
    inp = syn.make_linear(384, 1280, M, r=r, alpha=16.0, seed=8, workload="test", dy_std=1.0)
    W, A, B, X, dY = (t.to(dev).contiguous() for t in (inp.W, inp.A, inp.B, inp.X, inp.dY))
    qs = b.qlora_quantize_nf4(W)
    Y, T = b.qlora_linear_fwd(qs, X, A, B, inp.alpha, T_save=True)
    dX, dA, dB = b.qlora_linear_bwd(qs, X, A, B, inp.alpha, dY, T_saved=T)
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    Wd = oracle.bf16_bits_to_f32(oracle.dequantize_nf4_single(
        oracle.quantize_nf4_single(bf16_to_f32_np(inp.W)))).astype(np.float64)
    Xn, An, Bn, dYn = (bf16_to_f32_np(t).astype(np.float64) for t in (inp.X, inp.A, inp.B, inp.dY))
    s = oracle.lora_scale(inp.alpha, inp.r)
    Yr, _ = oracle.linear_fwd(Wd, Xn, An, Bn, s)
    dXr, dAr, dBr = oracle.linear_bwd(Wd, Xn, An, Bn, dYn, s)
    for name, got, want in (("Y", Y, Yr), ("dX", dX, dXr), ("dA", dA, dAr), ("dB", dB, dBr)):
        ok, err = gemm_close(bf16_to_f32_np(got), want)
        assert ok, (name, err)


def test_single_merge_bit_exact():
    dev = require_gpu()
    N, K = 100, 320
    W = syn.normal_bf16((N, K), 0.02, 4, "test", 140)
    ads = [(syn.normal_bf16((r, K), 0.02, 4, "test", 141 + 2 * i),
            syn.normal_bf16((N, r), 0.02, 4, "test", 142 + 2 * i)) for i, r in enumerate((8, 24))]
    alphas, weights = (16.0, 8.0), (0.7, -0.3)
    qs = b.qlora_quantize_nf4(W.to(dev))
    out = b.qlora_merge_lora(qs, [(A.to(dev), B.to(dev), al, wt) for (A, B), al, wt in zip(ads, alphas, weights)])
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    Wd = oracle.dequantize_nf4_single(oracle.quantize_nf4_single(bf16_to_f32_np(W)))
    spec = [(bf16_to_f32_np(A), bf16_to_f32_np(B), A.shape[0], al, wt) for (A, B), al, wt in zip(ads, alphas, weights)]
    assert np.array_equal(bf16_bits_np(out), oracle.merge_lora(Wd, spec))
