"""GPU parity of quantize + double quantization + dequantization against the
CPU oracle, through the C ABI. Codes, int8 constants, scales, the mean and the
dequantized bf16 weights must be bit-identical."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_absmax_b200 import binding as b
from bit_nf4_quantized_absmax_b200 import synthetic as syn
from tests.helpers import bf16_bits_np, bf16_to_f32_np, require_gpu

pytestmark = pytest.mark.gpu


def _gpu_quant(W_cpu: torch.Tensor):
    dev = require_gpu()
    W = W_cpu.to(dev).contiguous()
    q = b.qlora_quantize_nf4_dq(W)
    Wd = b.qlora_dequantize_nf4_dq(q)
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    return q, Wd


def _assert_bit_exact(W_cpu: torch.Tensor, q, Wd):
    Wf = bf16_to_f32_np(W_cpu)
    ref = oracle.quantize_nf4_dq(Wf)
    assert float(q.mean.cpu().numpy()[0]).hex() == float(ref.mean).hex()
    assert np.array_equal(q.dq_scale.cpu().numpy().view(np.uint32), ref.dq_scale.view(np.uint32))
    assert np.array_equal(q.absmax_q.cpu().numpy(), ref.absmax_q)
    got_packed = q.packed.cpu().numpy()
    if not np.array_equal(got_packed, ref.packed):
        bad = np.nonzero(got_packed != ref.packed)[0]
        raise AssertionError(f"{bad.size} packed bytes differ, first at {bad[:8]}")
    ref_wd = oracle.dequantize_nf4_dq(ref)
    assert np.array_equal(bf16_bits_np(Wd), ref_wd)


@pytest.mark.parametrize("shape", [(1024, 1024), (1, 64), (3, 192), (257, 320), (33, 64 * 300)])
def test_quantize_dequant_bit_exact_small(shape):
    W = syn.normal_bf16(shape, 0.02, 0, "test", shape[0] * 7 + shape[1])
    q, Wd = _gpu_quant(W)
    _assert_bit_exact(W, q, Wd)


def test_single_linear_workload_bit_exact():
    inp = syn.single_linear(0)
    q, Wd = _gpu_quant(inp.W)
    _assert_bit_exact(inp.W, q, Wd)


def test_edge_blocks():
    """All-zero blocks (codes 7), an all-equal group (s_g = 0), a ragged last
    group, huge and subnormal magnitudes, signed zeros."""
    W = syn.normal_bf16((40, 64 * 70), 0.02, 0, "test", 101).float()
    W[0, :64] = 0.0
    W[1, :] = 0.0
    W[2, 64:128] = -0.0
    W[3, :] = 0.03125                        # equal absmax everywhere in this row
    W[5, :64] *= 2.0 ** 100
    W[6, :64] *= 2.0 ** -120                 # bf16 subnormal range
    W[7, :64] = torch.tensor([2.0 ** -133] * 64)
    W[8, :] = 0.0625
    W[8, ::3] = -0.0625
    Wb = W.to(torch.bfloat16)
    q, Wd = _gpu_quant(Wb)
    _assert_bit_exact(Wb, q, Wd)


def test_all_equal_constants_group():
    """Every block has the same absmax: mean = that value, scales 0, codes 0."""
    W = torch.full((16, 64 * 64), 0.05, dtype=torch.bfloat16)
    W[:, ::2] = -0.05
    q, Wd = _gpu_quant(W)
    _assert_bit_exact(W, q, Wd)
    assert np.all(q.dq_scale.cpu().numpy() == 0)


def _ratio_tensor(seed=5):
    """Blocks holding every pair (w, m) of bf16 significands, with m the block
    absmax and w = +-sw * 2^(e_m - d), d = 0..10, at random absolute exponents.
    Covers every quotient the nearest-code decision can see."""
    rng = np.random.default_rng(seed)
    sig = (np.arange(128, dtype=np.float64) + 128.0) / 128.0  # 1.0 .. 1.9921875
    rows = []
    for sm in sig:
        vals = []
        for d in range(11):
            for sw in sig:
                if d == 0 and sw > sm:
                    continue
                vals.append(sw * 2.0 ** -d)
                vals.append(-sw * 2.0 ** -d)
        vals = np.array(vals)
        rng.shuffle(vals)
        nb = (len(vals) + 62) // 63
        vals = np.concatenate([vals, np.zeros(nb * 63 - len(vals))]).reshape(nb, 63)
        for blk in vals:
            e = int(rng.integers(-20, 8))
            pos = int(rng.integers(0, 64))
            full = np.insert(blk, pos, sm) * 2.0 ** e
            rows.append(full)
    A = np.stack(rows).astype(np.float32)
    n = A.shape[0] - A.shape[0] % 8
    return torch.from_numpy(A[:n].reshape(-1, 64 * 8)).to(torch.bfloat16)


def test_nearest_code_every_significand_pair():
    W = _ratio_tensor()
    # the construction is exact in bf16 (significands have 8 bits)
    q, Wd = _gpu_quant(W)
    _assert_bit_exact(W, q, Wd)


def test_student_t_heavy_tails_bit_exact():
    W = syn.student_t_bf16((512, 2048), 4, 0.02, 0, "test", 77)
    q, Wd = _gpu_quant(W)
    _assert_bit_exact(W, q, Wd)


@pytest.mark.parametrize("shape", syn.LLAMA7B_SHAPES)
def test_llama7b_shapes_full_size(shape):
    """Full-size 7B-shaped weights: constants, scales and mean compared in full;
    codes and dequantized values compared on a sample of 64 rows (the oracle
    computes rows one by one from the full-tensor mean)."""
    W = syn.normal_bf16(shape, 0.02, 0, "llama7b", 16 * syn.LLAMA7B_SHAPES.index(shape))
    q, Wd = _gpu_quant(W)
    Wf = bf16_to_f32_np(W)
    codes_absmax = np.max(np.abs(Wf.reshape(-1, 64)), axis=1)
    qq, sc, mu = oracle.double_quantize(codes_absmax)
    assert float(q.mean.cpu().numpy()[0]).hex() == float(mu).hex()
    assert np.array_equal(q.absmax_q.cpu().numpy(), qq)
    assert np.array_equal(q.dq_scale.cpu().numpy().view(np.uint32), sc.view(np.uint32))
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(shape[0], 64, replace=False))
    rows = np.concatenate([[0, shape[0] - 1], rows])
    cb = oracle.nf4_codebook()
    packed = q.packed.cpu().numpy().reshape(shape[0], shape[1] // 2)
    wd_bits = bf16_bits_np(Wd)
    kb = shape[1] // 64
    for rrow in rows:
        codes, am = oracle.quantize_nf4(Wf[rrow:rrow + 1], cb)
        assert np.array_equal(packed[rrow], oracle.nf4.pack_codes(codes))
        # the group index of a block is global: decode with the global scales
        mp = oracle.nf4.dequant_constants(qq, sc, mu)[rrow * kb:(rrow + 1) * kb]
        prod = (cb[codes.reshape(-1, 64)] * mp[:, None]).astype(np.float32)
        assert np.array_equal(wd_bits[rrow], oracle.f32_to_bf16_bits_rn(prod).reshape(-1))
