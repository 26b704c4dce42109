"""Both decode kernels (M <= 16) on the same cases: the X-resident kernel and
the TMA-ring kernel, each forced through QLORA_DECODE_RES (read by the library
on every call), against the fp64 oracle: ragged rows and K, ranks with
r % 16 == 8, 1..16 tokens, single-level storage, and repeated calls that must
give identical bits."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_absmax_b200 import binding as b
from bit_nf4_quantized_absmax_b200 import synthetic as syn
from tests.helpers import bf16_to_f32_np, gemm_close, require_gpu

pytestmark = pytest.mark.gpu

CASES = [  # (N, K, M, r)
    (1, 64, 1, 16), (17, 320, 9, 16), (100, 64, 16, 8), (40, 1088, 3, 24), (384, 1280, 4, 64),
    (136, 320, 16, 72), (1000, 4160, 1, 64), (2048, 4096, 8, 64), (4096, 4096, 16, 64), (3000, 256, 2, 32),
]


def _wd(W_cpu, single):
    Wf = bf16_to_f32_np(W_cpu)
    if single:
        return oracle.bf16_bits_to_f32(oracle.dequantize_nf4_single(oracle.quantize_nf4_single(Wf)))
    return oracle.bf16_bits_to_f32(oracle.dequantize_nf4_dq(oracle.quantize_nf4_dq(Wf)))


@pytest.mark.parametrize("mode", ["1", "0"])
def test_decode_kernel_cases(mode, monkeypatch):
    monkeypatch.setenv("QLORA_DECODE_RES", mode)
    dev = require_gpu()
    for i, (N, K, M, r) in enumerate(CASES):
        single = i % 3 == 2
        inp = syn.make_linear(N, K, M, r=r, alpha=16.0, seed=30 + i, workload="test", dy_std=1.0)
        W, A, B, X = (t.to(dev).contiguous() for t in (inp.W, inp.A, inp.B, inp.X))
        q = b.qlora_quantize_nf4(W) if single else b.qlora_quantize_nf4_dq(W)
        Y, T = b.qlora_linear_fwd(q, X, A, B, inp.alpha, T_save=True)
        Y2, _ = b.qlora_linear_fwd(q, X, A, B, inp.alpha)
        torch.cuda.synchronize()
        assert b.qlora_device_error() == 0
        assert torch.equal(Y, Y2), (mode, N, K, M)  # identical bits on a repeat
        Xn, An, Bn = (bf16_to_f32_np(t).astype(np.float64) for t in (inp.X, inp.A, inp.B))
        Yr, Tr = oracle.linear_fwd(_wd(inp.W, single).astype(np.float64), Xn, An, Bn,
                                   oracle.lora_scale(inp.alpha, inp.r))
        ok, err = gemm_close(bf16_to_f32_np(Y), Yr)
        assert ok, (mode, N, K, M, r, err)
        assert np.allclose(T.cpu().numpy(), Tr, rtol=1e-4, atol=1e-4 * np.abs(Tr).max())


DEFAULT_CASES = [  # (N, K, M, r): shapes the library's own choice sends to the X-resident kernel
    (8192, 2048, 8, 64),  # K < N, 2^24 entries: up to 8 tokens
    (2048, 2048, 4, 64),  # square, 2^22 entries: up to 4 tokens
    (2048, 2048, 2, 64),
]


def test_decode_default_choice_cases(monkeypatch):
    """The library's own kernel choice (no QLORA_DECODE_RES) on shapes past the
    crossover, against the fp64 oracle, with identical bits on a repeat."""
    monkeypatch.delenv("QLORA_DECODE_RES", raising=False)
    dev = require_gpu()
    for i, (N, K, M, r) in enumerate(DEFAULT_CASES):
        inp = syn.make_linear(N, K, M, r=r, alpha=16.0, seed=60 + i, workload="test", dy_std=1.0)
        W, A, B, X = (t.to(dev).contiguous() for t in (inp.W, inp.A, inp.B, inp.X))
        q = b.qlora_quantize_nf4_dq(W)
        Y, _ = b.qlora_linear_fwd(q, X, A, B, inp.alpha)
        Y2, _ = b.qlora_linear_fwd(q, X, A, B, inp.alpha)
        torch.cuda.synchronize()
        assert b.qlora_device_error() == 0
        assert torch.equal(Y, Y2), (N, K, M)
        Xn, An, Bn = (bf16_to_f32_np(t).astype(np.float64) for t in (inp.X, inp.A, inp.B))
        Yr, _ = oracle.linear_fwd(_wd(inp.W, False).astype(np.float64), Xn, An, Bn,
                                  oracle.lora_scale(inp.alpha, inp.r))
        ok, err = gemm_close(bf16_to_f32_np(Y), Yr)
        assert ok, (N, K, M, r, err)
