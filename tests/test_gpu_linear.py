"""GPU parity of the QLoRA linear forward and backward against the fp64 oracle,
through the C ABI. Outputs and gradients must be within 2e-3 relative
Frobenius error of the oracle evaluated with the same bf16 inputs and the same
dequantized weight W'."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_absmax_b200 import binding as b
from bit_nf4_quantized_absmax_b200 import synthetic as syn
from tests.helpers import bf16_to_f32_np, gemm_close, rel_fro, require_gpu

pytestmark = pytest.mark.gpu


def _oracle_wd(W_cpu):
    """W' computed by the oracle alone (quantize + double-quant + dequant)."""
    qw = oracle.quantize_nf4_dq(bf16_to_f32_np(W_cpu))
    return oracle.bf16_bits_to_f32(oracle.dequantize_nf4_dq(qw)).astype(np.float64)


_WD_CACHE = {}


def _oracle_wd_cached(key, W_cpu):
    if key not in _WD_CACHE:
        _WD_CACHE.clear()
        _WD_CACHE[key] = _oracle_wd(W_cpu)
    return _WD_CACHE[key]


def _run(inp: syn.LinearInputs, need_dX=True, use_saved_T=True):
    dev = require_gpu()
    W, A, B, X, dY = (t.to(dev).contiguous() for t in (inp.W, inp.A, inp.B, inp.X, inp.dY))
    q = b.qlora_quantize_nf4_dq(W)
    Y, T = b.qlora_linear_fwd(q, X, A, B, inp.alpha, T_save=True)
    dX, dA, dB = b.qlora_linear_bwd(q, X, A, B, inp.alpha, dY, T_saved=T if use_saved_T else None,
                                    need_dX=need_dX)
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    return Y, T, dX, dA, dB


def _check_full(inp: syn.LinearInputs, need_dX=True, use_saved_T=True):
    Y, T, dX, dA, dB = _run(inp, need_dX, use_saved_T)
    Wd = _oracle_wd(inp.W)
    X, A, B, dY = (bf16_to_f32_np(t).astype(np.float64) for t in (inp.X, inp.A, inp.B, inp.dY))
    s = oracle.lora_scale(inp.alpha, inp.r)
    Yr, Tr = oracle.linear_fwd(Wd, X, A, B, s)
    dXr, dAr, dBr = oracle.linear_bwd(Wd, X, A, B, dY, s)
    checks = {"Y": gemm_close(bf16_to_f32_np(Y), Yr), "dA": gemm_close(bf16_to_f32_np(dA), dAr),
              "dB": gemm_close(bf16_to_f32_np(dB), dBr)}
    if need_dX:
        checks["dX"] = gemm_close(bf16_to_f32_np(dX), dXr)
    errs = {k: v[1] for k, v in checks.items()}
    errs["T"] = rel_fro(T.cpu().numpy(), Tr)
    assert errs["T"] < 1e-5, errs
    assert all(v[0] for v in checks.values()), errs
    return errs


def test_single_linear_workload():
    """1024x1024, 16 tokens, r=16, alpha=16 (decode forward, tensor-core backward)."""
    _check_full(syn.single_linear(0))


@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_shapes_small(M):
    inp = syn.make_linear(384, 1280, M, r=64, alpha=16.0, seed=1, workload="test", dy_std=1.0)
    _check_full(inp)


@pytest.mark.parametrize("M,N,K,r", [(256, 512, 1024, 64), (200, 328, 320, 8), (130, 264, 576, 72),
                                     (17, 1000, 192, 24), (384, 2048, 512, 128)])
def test_tensor_core_shapes(M, N, K, r):
    """Several M/N tiles, ragged M, N and K tails, r below, at and above one 64-wide slab."""
    inp = syn.make_linear(N, K, M, r=r, alpha=16.0, seed=2, workload="test", dy_std=0.5)
    _check_full(inp)


@pytest.mark.parametrize("N,K", [(1, 64), (17, 320), (100, 64), (40, 1088)])
def test_decode_ragged(N, K):
    """Forward with row counts that are not a multiple of 16 and K that is not a
    multiple of 256; the backward rejects N % 8 != 0 before launching."""
    dev = require_gpu()
    for M in (1, 9, 16):
        inp = syn.make_linear(N, K, M, r=16, alpha=8.0, seed=3, workload="test", dy_std=1.0)
        W, A, B, X, dY = (t.to(dev) for t in (inp.W, inp.A, inp.B, inp.X, inp.dY))
        q = b.qlora_quantize_nf4_dq(W)
        Y, _ = b.qlora_linear_fwd(q, X, A, B, inp.alpha)
        torch.cuda.synchronize()
        Wd = _oracle_wd(inp.W)
        Xn, An, Bn = (bf16_to_f32_np(t).astype(np.float64) for t in (inp.X, inp.A, inp.B))
        Yr, _ = oracle.linear_fwd(Wd, Xn, An, Bn, oracle.lora_scale(inp.alpha, inp.r))
        assert gemm_close(bf16_to_f32_np(Y), Yr)[0]
        if N % 8:
            with pytest.raises(b.QloraError) as e:
                b.qlora_linear_bwd(q, X, A, B, inp.alpha, dY)
            assert e.value.status == 2
        else:
            _check_full(inp)
    assert b.qlora_device_error() == 0


@pytest.mark.parametrize("r", [8, 24, 72])
def test_decode_ranks_not_multiple_of_16(r):
    """Decode forward with r % 16 == 8: the LoRA-up runs in 16-rank steps, and the
    upper half of the last step lies outside the adapter. With W = 0 the output is
    the LoRA term alone (a zero weight dequantizes to exact zeros), so a wrong
    rank anywhere in it shows."""
    dev = require_gpu()
    for M in (1, 9, 16):
        inp = syn.make_linear(136, 320, M, r=r, alpha=16.0, seed=6, workload="test", dy_std=1.0)
        Xn, An, Bn = (bf16_to_f32_np(t).astype(np.float64) for t in (inp.X, inp.A, inp.B))
        s = oracle.lora_scale(inp.alpha, inp.r)
        for zero_w in (True, False):
            W = torch.zeros_like(inp.W) if zero_w else inp.W
            X, A, B = (t.to(dev).contiguous() for t in (inp.X, inp.A, inp.B))
            q = b.qlora_quantize_nf4_dq(W.to(dev))
            Y, T = b.qlora_linear_fwd(q, X, A, B, inp.alpha, T_save=True)
            torch.cuda.synchronize()
            Wd = np.zeros((136, 320)) if zero_w else _oracle_wd(inp.W)
            Yr, Tr = oracle.linear_fwd(Wd, Xn, An, Bn, s)
            ok, err = gemm_close(bf16_to_f32_np(Y), Yr)
            assert ok, (M, zero_w, err)
            assert rel_fro(T.cpu().numpy().astype(np.float64), Tr) < 1e-5
    assert b.qlora_device_error() == 0


def test_recomputed_T_matches_saved_T_path():
    inp = syn.make_linear(512, 768, 300, r=32, alpha=16.0, seed=4, workload="test", dy_std=0.5)
    _check_full(inp, use_saved_T=False)
    _check_full(inp, need_dX=False)


def test_empty_batch():
    dev = require_gpu()
    inp = syn.make_linear(64, 128, 0, r=16, alpha=16.0, seed=5, workload="test")
    W, A, B = (t.to(dev) for t in (inp.W, inp.A, inp.B))
    q = b.qlora_quantize_nf4_dq(W)
    X = torch.empty(0, 128, dtype=torch.bfloat16, device=dev)
    dY = torch.empty(0, 64, dtype=torch.bfloat16, device=dev)
    Y, _ = b.qlora_linear_fwd(q, X, A, B, 16.0)
    assert Y.shape == (0, 64)
    dA = torch.full((16, 128), 7.0, dtype=torch.bfloat16, device=dev)
    dB = torch.full((64, 16), 7.0, dtype=torch.bfloat16, device=dev)
    _, dA, dB = b.qlora_linear_bwd(q, X, A, B, 16.0, dY, need_dX=False, dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dA).item() == 0 and torch.count_nonzero(dB).item() == 0


@pytest.mark.parametrize("shape", syn.LLAMA7B_SHAPES)
def test_llama7b_decode_full_size(shape):
    """7B-shaped decode at M = 1, 4, 16: the oracle evaluates the full output."""
    N, K = shape
    for M in (1, 4, 16):
        inp = syn.make_linear(N, K, M, r=64, alpha=16.0, seed=0, workload="llama7b",
                              layer=syn.LLAMA7B_SHAPES.index(shape))
        dev = require_gpu()
        W, A, B, X = (t.to(dev) for t in (inp.W, inp.A, inp.B, inp.X))
        q = b.qlora_quantize_nf4_dq(W)
        Y, _ = b.qlora_linear_fwd(q, X, A, B, inp.alpha)
        torch.cuda.synchronize()
        Wd = _oracle_wd_cached(("llama7b", shape), inp.W)
        Xn, An, Bn = (bf16_to_f32_np(t).astype(np.float64) for t in (inp.X, inp.A, inp.B))
        Yr, _ = oracle.linear_fwd(Wd, Xn, An, Bn, oracle.lora_scale(inp.alpha, inp.r))
        ok, err = gemm_close(bf16_to_f32_np(Y), Yr)
        assert ok, (M, err)


@pytest.mark.parametrize("shape", syn.LLAMA7B_SHAPES)
def test_llama7b_train_full_size_sampled(shape):
    """M = 4096 training shapes in the launch configuration the benchmark times:
    Y and dX are checked on 48 sampled token rows (the oracle evaluates them row
    by row), dA and dB in full (their reduction runs over all tokens)."""
    N, K = shape
    M = 4096
    inp = syn.make_linear(N, K, M, r=64, alpha=16.0, seed=0, workload="llama7b_train",
                          layer=syn.LLAMA7B_SHAPES.index(shape))
    dev = require_gpu()
    W, A, B, X, dY = (t.to(dev) for t in (inp.W, inp.A, inp.B, inp.X, inp.dY))
    q = b.qlora_quantize_nf4_dq(W)
    Y, T = b.qlora_linear_fwd(q, X, A, B, inp.alpha, T_save=True)
    dX, dA, dB = b.qlora_linear_bwd(q, X, A, B, inp.alpha, dY, T_saved=T)
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    Wd = _oracle_wd(inp.W)
    Xn, An, Bn, dYn = (bf16_to_f32_np(t).astype(np.float64) for t in (inp.X, inp.A, inp.B, inp.dY))
    s = np.float64(oracle.lora_scale(inp.alpha, inp.r))
    rows = np.concatenate([[0, M - 1], np.random.default_rng(7).choice(M, 46, replace=False)])
    Yr, _ = oracle.linear_fwd(Wd, Xn[rows], An, Bn, s)
    assert gemm_close(bf16_to_f32_np(Y)[rows], Yr)[0]
    dXr, _, _ = oracle.linear_bwd(Wd, Xn[rows], An, Bn, dYn[rows], s)
    assert gemm_close(bf16_to_f32_np(dX)[rows], dXr)[0]
    U = dYn @ Bn
    dAr = s * (U.T @ Xn)
    dBr = s * (dYn.T @ (Xn @ An.T))
    assert gemm_close(bf16_to_f32_np(dA), dAr)[0]
    assert gemm_close(bf16_to_f32_np(dB), dBr)[0]
