"""Training forward and dX with the NF4 weight decoded inside the 2-CTA tcgen05
GEMMs ("QLoRA vs ChatGPT", capability 5: block-wise dequantization on the fly),
selected with QLORA_FWD_FUSED=1: the same W' bits and the same accumulation
order as the dequant-then-GEMM path, so Y, T, dX, dA and dB must be identical
bit for bit, and within the GEMM tolerance of the fp64 oracle."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_absmax_b200 import binding as b
from bit_nf4_quantized_absmax_b200 import synthetic as syn
from tests.helpers import bf16_to_f32_np, gemm_close, require_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K,r,single", [(256, 512, 1024, 64, False), (300, 328, 320, 8, False),
                                             (512, 264, 576, 72, True), (1024, 1000, 2048, 128, False),
                                             (4096, 11008, 4096, 64, False)])
def test_fused_forward_bit_identical(M, N, K, r, single, monkeypatch):
    dev = require_gpu()
    inp = syn.make_linear(N, K, M, r=r, alpha=16.0, seed=21, workload="test", dy_std=1.0)
    W, A, B, X, dY = (t.to(dev).contiguous() for t in (inp.W, inp.A, inp.B, inp.X, inp.dY))
    q = b.qlora_quantize_nf4(W) if single else b.qlora_quantize_nf4_dq(W)
    monkeypatch.setenv("QLORA_FWD_FUSED", "0")
    Y0, T0 = b.qlora_linear_fwd(q, X, A, B, inp.alpha, T_save=True)
    g0 = b.qlora_linear_bwd(q, X, A, B, inp.alpha, dY, T_saved=T0)
    monkeypatch.setenv("QLORA_FWD_FUSED", "1")
    Y1, T1 = b.qlora_linear_fwd(q, X, A, B, inp.alpha, T_save=True)
    Y2, _ = b.qlora_linear_fwd(q, X, A, B, inp.alpha)
    g1 = b.qlora_linear_bwd(q, X, A, B, inp.alpha, dY, T_saved=T1)
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    assert torch.equal(T0, T1)
    assert torch.equal(Y0, Y1) and torch.equal(Y1, Y2)
    for a0, a1 in zip(g0, g1):  # dX, dA, dB
        assert torch.equal(a0, a1)
    if N * K <= 4 << 20:
        Wf = bf16_to_f32_np(inp.W)
        wd = (oracle.dequantize_nf4_single(oracle.quantize_nf4_single(Wf)) if single
              else oracle.dequantize_nf4_dq(oracle.quantize_nf4_dq(Wf)))
        Xn, An, Bn = (bf16_to_f32_np(t).astype(np.float64) for t in (inp.X, inp.A, inp.B))
        Yr, _ = oracle.linear_fwd(oracle.bf16_bits_to_f32(wd).astype(np.float64), Xn, An, Bn,
                                  oracle.lora_scale(inp.alpha, inp.r))
        ok, err = gemm_close(bf16_to_f32_np(Y1), Yr)
        assert ok, err
