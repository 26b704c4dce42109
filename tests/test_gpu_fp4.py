"""GPU parity of the FP4 data type (the Float4 that the QLoRA errata page's
findings on the paper's p.8 Table 4 compare with NFloat4), through the C ABI:
the library's quantize and dequant kernels with the FP4 table give the oracle's
codes, constants and dequantized bf16 weights bit for bit, in both storage
kinds, and the NF4 path of the same entry points equals the NF4 calls."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_absmax_b200 import binding as b
from bit_nf4_quantized_absmax_b200 import synthetic as syn
from tests.helpers import bf16_bits_np, bf16_to_f32_np, require_gpu
from tests.test_gpu_quant import _ratio_tensor

pytestmark = pytest.mark.gpu


def _check(W_cpu: torch.Tensor, double_quant: bool):
    dev = require_gpu()
    W = W_cpu.to(dev).contiguous()
    q = b.qlora_quantize_4bit(W, b.DTYPE_FP4, double_quant=double_quant)
    Wd = b.qlora_dequantize_4bit(q, b.DTYPE_FP4)
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    cb = oracle.fp4_codebook()
    Wf = bf16_to_f32_np(W_cpu)
    if double_quant:
        ref = oracle.quantize_nf4_dq(Wf, cb)
        assert float(q.mean.cpu().numpy()[0]).hex() == float(ref.mean).hex()
        assert np.array_equal(q.dq_scale.cpu().numpy().view(np.uint32), ref.dq_scale.view(np.uint32))
        assert np.array_equal(q.absmax_q.cpu().numpy(), ref.absmax_q)
        ref_wd = oracle.dequantize_nf4_dq(ref, cb)
    else:
        ref = oracle.quantize_nf4_single(Wf, cb)
        assert np.array_equal(q.absmax.cpu().numpy().view(np.uint32), ref.absmax.view(np.uint32))
        ref_wd = oracle.dequantize_nf4_single(ref, cb)
    got = q.packed.cpu().numpy()
    if not np.array_equal(got, ref.packed):
        bad = np.nonzero(got != ref.packed)[0]
        raise AssertionError(f"{bad.size} packed bytes differ, first at {bad[:8]}")
    assert np.array_equal(bf16_bits_np(Wd), ref_wd)
    codes = oracle.unpack_codes(got)
    assert 15 not in np.unique(codes).tolist()  # the repeated +1 is never selected
    return q


@pytest.mark.parametrize("double_quant", [True, False])
@pytest.mark.parametrize("shape", [(1024, 1024), (3, 192), (257, 320)])
def test_fp4_bit_exact(shape, double_quant):
    W = syn.normal_bf16(shape, 0.02, 0, "test", 3 * shape[0] + shape[1])
    _check(W, double_quant)


def test_fp4_every_significand_pair_and_heavy_tails():
    _check(_ratio_tensor(seed=9), True)
    _check(syn.student_t_bf16((256, 2048), 4, 0.02, 0, "test", 78), True)


def test_fp4_edge_blocks():
    W = syn.normal_bf16((12, 64 * 40), 0.02, 0, "test", 201).float()
    W[0, :64] = 0.0
    W[2, 64:128] = -0.0
    W[3, :] = 0.03125
    W[5, :64] *= 2.0 ** 100
    W[6, :64] *= 2.0 ** -120
    _check(W.to(torch.bfloat16), True)
    _check(W.to(torch.bfloat16), False)


def test_nf4_through_the_dtype_calls_equals_nf4_calls():
    dev = require_gpu()
    W = syn.normal_bf16((512, 1024), 0.02, 0, "test", 202).to(dev)
    q1 = b.qlora_quantize_nf4_dq(W)
    q2 = b.qlora_quantize_4bit(W, b.DTYPE_NF4)
    for name in ("packed", "absmax_q", "dq_scale", "mean"):
        assert torch.equal(getattr(q1, name), getattr(q2, name))
    assert torch.equal(b.qlora_dequantize_nf4_dq(q1), b.qlora_dequantize_4bit(q2, b.DTYPE_NF4))
    # FP4 and NF4 differ on the same weight (the tables are not the same)
    q3 = b.qlora_quantize_4bit(W, b.DTYPE_FP4)
    assert not torch.equal(q1.packed, q3.packed)
