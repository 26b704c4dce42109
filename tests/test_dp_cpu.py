"""Data-parallel exchange of the LoRA gradients on CPU: world size 2 over gloo.

Each rank computes the gradients of its own token shard (here with the fp64
oracle, rounded to fp32 as qlora_linear_bwd_f32 returns them, standing in for
the kernels that need a GPU) and calls the module's all-reduce; both ranks must
end with the same dA and dB, equal to the full-batch gradients within the
GEMM tolerance."""
from __future__ import annotations

import datetime
import json
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    sys.path.insert(0, ROOT)
    from bit_nf4_quantized_absmax_b200 import synthetic as syn
    return syn.make_linear(96, 192, 50, r=16, alpha=16.0, seed=12, workload="test", dy_std=1.0)


def _oracle_grads(inp, rows):
    import oracle
    from tests.helpers import bf16_to_f32_np
    qw = oracle.quantize_nf4_dq(bf16_to_f32_np(inp.W))
    Wd = oracle.bf16_bits_to_f32(oracle.dequantize_nf4_dq(qw)).astype(np.float64)
    X, A, B, dY = (bf16_to_f32_np(t).astype(np.float64) for t in (inp.X, inp.A, inp.B, inp.dY))
    _, dA, dB = oracle.linear_bwd(Wd, X[rows], A, B, dY[rows], oracle.lora_scale(inp.alpha, inp.r))
    return dA, dB


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from bit_nf4_quantized_absmax_b200 import dp
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    inp = _case()
    sl = dp.shard_tokens(inp.X.shape[0], rank, world)
    dA_l, dB_l = _oracle_grads(inp, sl)
    # fp32, in the flat layout qlora_linear_bwd_dp writes (dA then dB)
    buf, vA, vB = dp.flat_grads(inp.r, inp.X.shape[1], inp.W.shape[0])
    vA.copy_(torch.from_numpy(dA_l.astype(np.float32)))
    vB.copy_(torch.from_numpy(dB_l.astype(np.float32)))
    dp.allreduce_grads(buf)
    dist.barrier()
    dist.destroy_process_group()
    # the one rounding to bf16 (the library's qlora_round_bf16 on a GPU); here torch's
    dA, dB = vA.to(torch.bfloat16), vB.to(torch.bfloat16)
    np.save(os.path.join(out_dir, f"dA{rank}.npy"), dA.float().numpy())
    np.save(os.path.join(out_dir, f"dB{rank}.npy"), dB.float().numpy())
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"lo": sl.start, "hi": sl.stop}, f)


def test_lora_gradients_summed_over_two_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    sys.path.insert(0, ROOT)
    from tests.helpers import gemm_close
    inp = _case()
    spans = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(world)]
    assert spans[0]["lo"] == 0 and spans[0]["hi"] == spans[1]["lo"] and spans[1]["hi"] == inp.X.shape[0]
    dA0, dA1 = (np.load(tmp_path / f"dA{r}.npy") for r in range(world))
    dB0, dB1 = (np.load(tmp_path / f"dB{r}.npy") for r in range(world))
    assert np.array_equal(dA0, dA1) and np.array_equal(dB0, dB1)  # every rank holds the same sums
    dA_ref, dB_ref = _oracle_grads(inp, slice(0, inp.X.shape[0]))
    assert gemm_close(dA0, dA_ref)[0] and gemm_close(dB0, dB_ref)[0]


def test_shard_tokens_cover_every_token_once():
    sys.path.insert(0, ROOT)
    from bit_nf4_quantized_absmax_b200 import dp
    for M in (0, 1, 7, 4096, 4097):
        for world in (1, 2, 3, 8):
            got = []
            for r in range(world):
                s = dp.shard_tokens(M, r, world)
                assert 0 <= s.stop - s.start <= M // world + 1
                got.extend(range(s.start, s.stop))
            assert got == list(range(M))
