"""Every entry point captured into one CUDA graph (as the benchmark times the
step) and replayed: the outputs equal those of eager calls bit for bit (the
kernels are deterministic and take their tensor maps by value, so a captured
launch is self-contained)."""
from __future__ import annotations

import pytest
import torch

from bit_nf4_quantized_absmax_b200 import binding as b
from bit_nf4_quantized_absmax_b200 import synthetic as syn
from tests.helpers import require_gpu

pytestmark = pytest.mark.gpu


def test_graph_replay_matches_eager():
    dev = require_gpu()
    inp = syn.make_linear(512, 768, 300, r=32, alpha=16.0, seed=21, workload="test", dy_std=0.5)
    W, A, B, X, dY = (t.to(dev).contiguous() for t in (inp.W, inp.A, inp.B, inp.X, inp.dY))
    Xd = X[:4].contiguous()
    q = b.NF4Weight.empty(512, 768, dev)
    qs = b.SingleNF4Weight.empty(512, 768, dev)
    outs = {k: torch.empty(s, dtype=torch.bfloat16, device=dev) for k, s in
            (("Wd", (512, 768)), ("Yd", (4, 512)), ("Y", (300, 512)), ("dX", (300, 768)), ("dA", (32, 768)),
             ("dB", (512, 32)), ("Wds", (512, 768)))}
    T = torch.empty(300, 32, dtype=torch.float32, device=dev)
    p32 = torch.linspace(-0.1, 0.1, 4096, device=dev)
    g16 = (torch.arange(4096, device=dev, dtype=torch.float32) * 1e-5).to(torch.bfloat16)
    m, v = torch.zeros(4096, device=dev), torch.zeros(4096, device=dev)
    ws = {k: torch.empty(64 << 20, dtype=torch.uint8, device=dev) for k in ("q", "dec", "fwd", "bwd")}

    def step():
        b.qlora_quantize_nf4_dq(W, out=q, workspace=ws["q"])
        b.qlora_quantize_nf4(W, out=qs)
        b.qlora_dequantize_nf4(q, out=outs["Wd"])
        b.qlora_dequantize_nf4(qs, out=outs["Wds"])
        b.qlora_linear_fwd(q, Xd, A, B, inp.alpha, Y=outs["Yd"], workspace=ws["dec"])
        b.qlora_linear_fwd(q, X, A, B, inp.alpha, Y=outs["Y"], T_save=T, workspace=ws["fwd"])
        b.qlora_linear_bwd(q, X, A, B, inp.alpha, dY, T_saved=T, dX=outs["dX"], dA=outs["dA"], dB=outs["dB"],
                           workspace=ws["bwd"])
        b.qlora_adamw_step(p32, g16, m, v, 1, weight_decay=0.01)

    p0 = p32.clone()
    step()
    torch.cuda.synchronize()
    eager = {k: t.clone() for k, t in outs.items()}
    eager.update(T=T.clone(), p=p32.clone(), m=m.clone(), v=v.clone(), packed=q.packed.clone(),
                 absmax=qs.absmax.clone())
    # reset the optimizer state so the replay repeats the same first step
    p32.copy_(p0)
    m.zero_()
    v.zero_()
    for t in list(outs.values()) + [T, q.packed, qs.absmax]:
        t.zero_()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        step()
    g.replay()
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    got = dict(outs, T=T, p=p32, m=m, v=v, packed=q.packed, absmax=qs.absmax)
    for k, ref in eager.items():
        assert torch.equal(got[k], ref), k


def test_graph_replays_split_tail_tiles():
    """A forward whose large GEMM splits its tiles in two along K (a reduction
    of 8192 over two tiles; the backward's dX GEMM, a reduction of 512, keeps
    whole tiles): the halves meet through flags that carry a tag of the launch,
    so repeated replays of one captured launch must give the eager bits every
    time, and the results must match the oracle."""
    import numpy as np

    import oracle
    from tests.helpers import bf16_to_f32_np, gemm_close

    dev = require_gpu()
    N, K, M = 512, 8192, 256  # one M tile, two N tiles: every tile is split
    inp = syn.make_linear(N, K, M, r=16, alpha=16.0, seed=23, workload="test", dy_std=0.5)
    W, A, B, X, dY = (t.to(dev).contiguous() for t in (inp.W, inp.A, inp.B, inp.X, inp.dY))
    q = b.qlora_quantize_nf4_dq(W)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dA = torch.empty(16, K, dtype=torch.bfloat16, device=dev)
    dB = torch.empty(N, 16, dtype=torch.bfloat16, device=dev)
    T = torch.empty(M, 16, dtype=torch.float32, device=dev)
    ws_f = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ws_b = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        b.qlora_linear_fwd(q, X, A, B, inp.alpha, Y=Y, T_save=T, workspace=ws_f)
        b.qlora_linear_bwd(q, X, A, B, inp.alpha, dY, T_saved=T, dX=dX, dA=dA, dB=dB, workspace=ws_b)

    step()
    torch.cuda.synchronize()
    eager_y, eager_dx = Y.clone(), dX.clone()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        step()
    for _ in range(3):
        Y.zero_()
        dX.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert b.qlora_device_error() == 0
        assert torch.equal(Y, eager_y)
        assert torch.equal(dX, eager_dx)
    Wd = oracle.bf16_bits_to_f32(oracle.dequantize_nf4_dq(oracle.quantize_nf4_dq(bf16_to_f32_np(inp.W))))
    Xn, An, Bn, dYn = (bf16_to_f32_np(t).astype(np.float64) for t in (inp.X, inp.A, inp.B, inp.dY))
    s = oracle.lora_scale(inp.alpha, inp.r)
    Yr, _ = oracle.linear_fwd(Wd.astype(np.float64), Xn, An, Bn, s)
    ok, err = gemm_close(bf16_to_f32_np(eager_y), Yr)
    assert ok, err
    dXr = oracle.linear_bwd(Wd.astype(np.float64), Xn, An, Bn, dYn, s)[0]
    ok, err = gemm_close(bf16_to_f32_np(eager_dx), dXr)
    assert ok, err
