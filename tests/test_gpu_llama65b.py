"""GPU parity on the Llama-65B-shaped workloads, through the C ABI:

* the three 65B linear shapes with heavy-tailed Student-t(4) weights (std 0.02):
  quantize + DQ, training forward/backward at M = 2048 and decode at M = 1;
* the whole-model sweep: 80 layers x 7 linears (64.76e9 weights) drawn on the
  device layer by layer into one reused buffer, quantized into resident NF4
  storage (~33.4 GB), then a dequant pass and an M = 1 decode pass over all 560
  linears; sampled linears are checked against the oracle.

Weights are drawn on the device by torch's seeded generator (too large for the
host); the oracle receives copies of the same bf16 values.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_absmax_b200 import binding as b
from bit_nf4_quantized_absmax_b200 import synthetic as syn
from tests.helpers import bf16_bits_np, bf16_to_f32_np, gemm_close, require_gpu

pytestmark = pytest.mark.gpu


def _oracle_quant(Wf: np.ndarray):
    """Oracle constants for the whole tensor (absmax is cheap), codes for all rows."""
    return oracle.quantize_nf4_dq(Wf)


def _check_constants_and_rows(q, ref, rows, K):
    assert float(q.mean.cpu().numpy()[0]).hex() == float(ref.mean).hex()
    assert np.array_equal(q.absmax_q.cpu().numpy(), ref.absmax_q)
    assert np.array_equal(q.dq_scale.cpu().numpy().view(np.uint32), ref.dq_scale.view(np.uint32))
    packed = q.packed.cpu().numpy().reshape(-1, K // 2)
    ref_packed = ref.packed.reshape(-1, K // 2)
    assert np.array_equal(packed[rows], ref_packed[rows])


@pytest.mark.parametrize("li", [0, 1, 2])
def test_llama65b_student_t_train_and_decode(li):
    dev = require_gpu()
    N, K = syn.LLAMA65B_SHAPES[li]
    M, r, alpha = 2048, 64, 16.0
    W = syn.student_t_bf16_device((N, K), 4, 0.02, 0, "llama65b", 16 * li, device=dev)
    A = syn.normal_bf16((r, K), 0.02, 0, "llama65b", 16 * li + 1).to(dev)
    B = syn.normal_bf16((N, r), 0.02, 0, "llama65b", 16 * li + 2).to(dev)
    X = syn.normal_bf16((M, K), 1.0, 0, "llama65b", 16 * li + 3).to(dev)
    dY = syn.normal_bf16((M, N), 0.01, 0, "llama65b", 16 * li + 4).to(dev)
    q = b.qlora_quantize_nf4_dq(W)
    Wd_gpu = b.qlora_dequantize_nf4_dq(q)
    Y, T = b.qlora_linear_fwd(q, X, A, B, alpha, T_save=True)
    Y1, _ = b.qlora_linear_fwd(q, X[:1].contiguous(), A, B, alpha)
    dX, dA, dB = b.qlora_linear_bwd(q, X, A, B, alpha, dY, T_saved=T)
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0

    Wf = bf16_to_f32_np(W)
    ref = _oracle_quant(Wf)
    rng = np.random.default_rng(li)
    rows = np.concatenate([[0, N - 1], rng.choice(N, 30, replace=False)])
    _check_constants_and_rows(q, ref, rows, K)
    wd_ref_bits = oracle.dequantize_nf4_dq(ref)
    assert np.array_equal(bf16_bits_np(Wd_gpu), wd_ref_bits)

    Wd = oracle.bf16_bits_to_f32(wd_ref_bits).astype(np.float64)
    Xn, An, Bn, dYn = (bf16_to_f32_np(t).astype(np.float64) for t in (X, A, B, dY))
    s = np.float64(oracle.lora_scale(alpha, r))
    mrows = np.concatenate([[0, M - 1], rng.choice(M, 22, replace=False)])
    Yr, _ = oracle.linear_fwd(Wd, Xn[mrows], An, Bn, s)
    assert gemm_close(bf16_to_f32_np(Y)[mrows], Yr)[0]
    assert gemm_close(bf16_to_f32_np(Y1), Yr[:1])[0]
    dXr, _, _ = oracle.linear_bwd(Wd, Xn[mrows], An, Bn, dYn[mrows], s)
    assert gemm_close(bf16_to_f32_np(dX)[mrows], dXr)[0]
    U = dYn @ Bn
    assert gemm_close(bf16_to_f32_np(dA), s * (U.T @ Xn))[0]
    assert gemm_close(bf16_to_f32_np(dB), s * (dYn.T @ (Xn @ An.T)))[0]


def test_llama65b_whole_model_sweep():
    dev = require_gpu()
    free, _ = torch.cuda.mem_get_info()
    assert free > 40e9, "the sweep keeps ~33.4 GB of NF4 storage resident"
    r, alpha = 64, 16.0
    shapes = syn.LLAMA65B_LAYER
    nmax = max(n * k for n, k in shapes)
    wbuf = torch.empty(nmax, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(64 << 20, dtype=torch.uint8, device=dev)
    stor, total_bytes = [], 0
    sampled = {(0, 0), (37, 5), (79, 6)}
    kept = {}
    for layer in range(syn.LLAMA65B_LAYERS):
        for j, (N, K) in enumerate(shapes):
            tid = 16 * (len(shapes) * layer + j)
            Wv = wbuf[:N * K].view(N, K)
            syn.normal_bf16_device((N, K), 0.02, 0, "sweep65b", tid, device=dev, out=Wv)
            q = b.qlora_quantize_nf4_dq(Wv, workspace=ws)
            stor.append(q)
            total_bytes += sum(t.numel() * t.element_size() for t in (q.packed, q.absmax_q, q.dq_scale, q.mean))
            if (layer, j) in sampled:
                kept[(layer, j)] = Wv.cpu()
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    # storage: 0.515869 B/param, 64.76e9 weights -> 33.4 GB (fits the 48 GB GPU of the pages)
    assert abs(total_bytes / 64.76005376e9 - 0.515869) < 1e-4
    assert 33.0e9 < total_bytes < 33.8e9

    # dequant pass and M = 1 decode pass over all 560 linears
    A_l, B_l, X_l, Y_l = [], [], [], []
    for j, (N, K) in enumerate(shapes):
        A_l.append(syn.normal_bf16((r, K), 0.02, 0, "sweep65b", 9000 + 4 * j).to(dev))
        B_l.append(syn.normal_bf16((N, r), 0.02, 0, "sweep65b", 9001 + 4 * j).to(dev))
        X_l.append(syn.normal_bf16((1, K), 1.0, 0, "sweep65b", 9002 + 4 * j).to(dev))
    outs, dq_kept = {}, {}
    dq_out = wbuf
    for i, q in enumerate(stor):
        layer, j = divmod(i, len(shapes))
        N, K = shapes[j]
        b.qlora_dequantize_nf4_dq(q, out=dq_out[:N * K].view(N, K))
        Y, _ = b.qlora_linear_fwd(q, X_l[j], A_l[j], B_l[j], alpha, workspace=ws)
        if (layer, j) in sampled:
            outs[(layer, j)] = Y
            dq_kept[(layer, j)] = dq_out[:N * K].view(N, K).cpu()
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0

    for (layer, j), Wc in kept.items():
        N, K = shapes[j]
        q = stor[len(shapes) * layer + j]
        ref = oracle.quantize_nf4_dq(bf16_to_f32_np(Wc))
        rows = np.concatenate([[0, N - 1], np.random.default_rng(layer).choice(N, 14, replace=False)])
        _check_constants_and_rows(q, ref, rows, K)
        wd_bits = oracle.dequantize_nf4_dq(ref)
        # the sweep's own dequant pass of this linear, bit for bit
        assert np.array_equal(bf16_bits_np(dq_kept[(layer, j)]), wd_bits)
        Wd = oracle.bf16_bits_to_f32(wd_bits).astype(np.float64)
        Yr, _ = oracle.linear_fwd(Wd, bf16_to_f32_np(X_l[j]).astype(np.float64),
                                  bf16_to_f32_np(A_l[j]).astype(np.float64),
                                  bf16_to_f32_np(B_l[j]).astype(np.float64), oracle.lora_scale(alpha, r))
        assert gemm_close(bf16_to_f32_np(outs[(layer, j)]), Yr)[0]
