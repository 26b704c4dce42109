"""Data-parallel step on the GPU kernels: per-shard backward passes summed in
fp32 (what the all-reduce does) give the full-batch LoRA gradients, and the
module runs through a real NCCL process group (world size 1 on one GPU; the
two-rank exchange itself is covered on CPU over gloo)."""
from __future__ import annotations

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from bit_nf4_quantized_absmax_b200 import binding as b
from bit_nf4_quantized_absmax_b200 import dp
from bit_nf4_quantized_absmax_b200 import synthetic as syn
from tests.helpers import bf16_to_f32_np, gemm_close, require_gpu

pytestmark = pytest.mark.gpu


def test_shard_gradients_sum_to_the_full_batch():
    dev = require_gpu()
    inp = syn.make_linear(512, 768, 600, r=32, alpha=16.0, seed=14, workload="test", dy_std=0.5)
    W, A, B, X, dY = (t.to(dev).contiguous() for t in (inp.W, inp.A, inp.B, inp.X, inp.dY))
    q = b.qlora_quantize_nf4_dq(W)
    world = 3
    dA_sum = torch.zeros(A.shape, dtype=torch.float32, device=dev)
    dB_sum = torch.zeros(B.shape, dtype=torch.float32, device=dev)
    for r in range(world):
        sl = dp.shard_tokens(X.shape[0], r, world)
        Xs, dYs = X[sl].contiguous(), dY[sl].contiguous()
        Y, T = dp.dp_linear_fwd(q, Xs, A, B, inp.alpha)
        _, dA32, dB32 = b.qlora_linear_bwd(q, Xs, A, B, inp.alpha, dYs, T_saved=T, grads_fp32=True)
        dA_sum += dA32  # what the all-reduce does across ranks
        dB_sum += dB32
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    Wd = oracle.bf16_bits_to_f32(oracle.dequantize_nf4_dq(oracle.quantize_nf4_dq(bf16_to_f32_np(inp.W))))
    Xn, An, Bn, dYn = (bf16_to_f32_np(t).astype(np.float64) for t in (inp.X, inp.A, inp.B, inp.dY))
    _, dAr, dBr = oracle.linear_bwd(Wd.astype(np.float64), Xn, An, Bn, dYn, oracle.lora_scale(inp.alpha, inp.r))
    assert gemm_close(dA_sum.cpu().numpy(), dAr)[0] and gemm_close(dB_sum.cpu().numpy(), dBr)[0]


def test_nccl_world_of_one():
    dev = require_gpu()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=dev)
    try:
        inp = syn.make_linear(256, 512, 64, r=16, alpha=16.0, seed=15, workload="test", dy_std=1.0)
        W, A, B, X, dY = (t.to(dev).contiguous() for t in (inp.W, inp.A, inp.B, inp.X, inp.dY))
        q = b.qlora_quantize_nf4_dq(W)
        Y, T = dp.dp_linear_fwd(q, X, A, B, inp.alpha)
        dX, dA, dB = dp.dp_linear_bwd(q, X, A, B, inp.alpha, dY, T_local=T)
        dX1, dA1, dB1 = b.qlora_linear_bwd(q, X, A, B, inp.alpha, dY, T_saved=T)
        torch.cuda.synchronize()
        # one rank: the fp32 gradients rounded once equal the bf16 backward bit for bit
        assert torch.equal(dA, dA1) and torch.equal(dB, dB1) and torch.equal(dX, dX1)
    finally:
        dist.destroy_process_group()


def test_bwd_dp_flat_buffer_event_and_rounding():
    """qlora_linear_bwd_dp: the flat fp32 buffer holds the bits of
    qlora_linear_bwd_f32's dA and dB, the event fires after them (a side stream
    that waits on it reads the finished gradients while dX runs), dX is the
    regular backward's, and qlora_round_bf16 of the buffer gives the bf16
    backward's gradients bit for bit."""
    dev = require_gpu()
    inp = syn.make_linear(1024, 512, 300, r=24, alpha=16.0, seed=16, workload="test", dy_std=1.0)
    W, A, B, X, dY = (t.to(dev).contiguous() for t in (inp.W, inp.A, inp.B, inp.X, inp.dY))
    q = b.qlora_quantize_nf4_dq(W)
    _, T = b.qlora_linear_fwd(q, X, A, B, inp.alpha, T_save=True)
    dX1, dA32, dB32 = b.qlora_linear_bwd(q, X, A, B, inp.alpha, dY, T_saved=T, grads_fp32=True)
    _, dA1, dB1 = b.qlora_linear_bwd(q, X, A, B, inp.alpha, dY, T_saved=T)
    r, N, K = inp.r, q.rows, q.cols
    grads, vA, vB = dp.flat_grads(r, K, N, device=dev)
    grads.fill_(float("nan"))
    ready = torch.cuda.Event()
    dX = b.qlora_linear_bwd_dp(q, X, A, B, inp.alpha, dY, grads, T_saved=T, grads_ready=ready)
    side = torch.cuda.Stream()
    side.wait_event(ready)
    with torch.cuda.stream(side):
        snap = grads.clone()                      # what an exchange on the side stream would read
        out, oA, oB = dp.flat_grads(r, K, N, device=dev, dtype=torch.bfloat16)
        b.qlora_round_bf16(grads, out, stream=side)
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    assert torch.equal(vA, dA32) and torch.equal(vB, dB32)
    assert torch.equal(snap, grads)
    assert torch.equal(dX, dX1)
    assert torch.equal(oA, dA1) and torch.equal(oB, dB1)
    # rounding of odd sizes and offsets (scalar tail, unaligned vector path)
    src = torch.randn(1003, device=dev)
    for off in (0, 1, 3):
        got = b.qlora_round_bf16(src[off:].contiguous())
        assert torch.equal(got, src[off:].to(torch.bfloat16))
    dst = torch.empty(1001, dtype=torch.bfloat16, device=dev)
    b.qlora_round_bf16(src[2:], dst[:1001])
    torch.cuda.synchronize()
    assert torch.equal(dst, src[2:].to(torch.bfloat16))

