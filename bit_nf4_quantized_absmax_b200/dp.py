"""Data-parallel QLoRA training step across ranks (one process per GPU).

Every rank holds the same frozen weight (its own NF4 copy: quantization is a
fixed function of the weight, so the copies are bit-identical without any
exchange) and the same LoRA parameters, and processes its own shard of the
tokens. The forward needs nothing from other ranks and dX stays with the rank
that owns the tokens; the only exchange is the sum of the LoRA gradients dA
and dB over ranks: each rank's backward returns them in fp32
(qlora_linear_bwd_f32), one all-reduce of a flat fp32 buffer sums them (NCCL
over NVLink on GPUs; any torch.distributed backend works) and the sums are
rounded once to bf16, as a single-GPU backward rounds its own. The compute
runs in the library's kernels through `binding`; this module only marshals
buffers and issues the collective.

("QLoRA vs ChatGPT", capability 5: gradients are computed only for the LoRA
parameters, which is what makes the exchange small: r (K + N) values per
linear.)

A weight too large to quantize on one rank can instead be quantized in row
shards (quantize_nf4_dq_sharded): each rank codes its rows, and the only
exchange is the exact sum of the block constants for the double-quantization
mean, as 256 integer bin totals ("Guanaco", "Core Architecture & Training":
the constants are quantized again, mean-centred). The shards' outputs are
bit-identical to quantizing the whole weight on one GPU.
"""
from __future__ import annotations

import math

import torch
import torch.distributed as dist

from . import binding


def allreduce_lora_grads(dA: torch.Tensor, dB: torch.Tensor, group=None,
                         out_A: torch.Tensor | None = None, out_B: torch.Tensor | None = None):
    """Sum the fp32 gradients dA and dB of this rank's token shard over the ranks
    of `group` (in place, one all-reduce of a flat fp32 buffer), then round the
    sums once into out_A / out_B when given (e.g. bf16 for the optimizer).
    Returns (dA, dB) or (out_A, out_B)."""
    assert dA.dtype == torch.float32 and dB.dtype == torch.float32
    nA = dA.numel()
    buf = torch.empty(nA + dB.numel(), dtype=torch.float32, device=dA.device)
    buf[:nA].copy_(dA.reshape(-1))
    buf[nA:].copy_(dB.reshape(-1))
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
    dA.copy_(buf[:nA].view_as(dA))
    dB.copy_(buf[nA:].view_as(dB))
    if out_A is None:
        return dA, dB
    out_A.copy_(dA)
    out_B.copy_(dB)
    return out_A, out_B


def dp_linear_fwd(q, X_local: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float, **kw):
    """Forward of this rank's token shard (no exchange). Returns (Y_local, T_local)."""
    return binding.qlora_linear_fwd(q, X_local, A, B, alpha, T_save=True, **kw)


def dp_linear_bwd(q, X_local: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float, dY_local: torch.Tensor,
                  T_local: torch.Tensor | None = None, need_dX: bool = True, group=None, **kw):
    """Backward of this rank's token shard with fp32 LoRA gradients
    (qlora_linear_bwd_f32), summed over ranks in fp32 and rounded once to bf16.
    Returns (dX_local or None, dA, dB), dA and dB bf16 and equal on every rank."""
    dX, dA32, dB32 = binding.qlora_linear_bwd(q, X_local, A, B, alpha, dY_local, T_saved=T_local, need_dX=need_dX,
                                              grads_fp32=True, **kw)
    dA = torch.empty(dA32.shape, dtype=torch.bfloat16, device=dA32.device)
    dB = torch.empty(dB32.shape, dtype=torch.bfloat16, device=dB32.device)
    allreduce_lora_grads(dA32, dB32, group, dA, dB)
    return dX, dA, dB


def shard_tokens(M: int, rank: int, world: int) -> slice:
    """Contiguous token range of a rank: sizes differ by at most one."""
    lo = rank * M // world
    hi = (rank + 1) * M // world
    return slice(lo, hi)


def group_aligned_rows(cols: int) -> int:
    """Smallest row count whose blocks fill whole 256-constant groups
    (rows * cols a multiple of 256 * 64 weights)."""
    return 16384 // math.gcd(16384, cols)


def shard_rows(total_rows: int, cols: int, rank: int, world: int) -> slice:
    """Row range of a rank for sharded quantization: boundaries on whole
    256-constant groups, sizes as even as that allows (the last shard takes the
    ragged end; a shard may be empty)."""
    u = group_aligned_rows(cols)
    units = -(-total_rows // u)
    lo = min(total_rows, (rank * units // world) * u)
    hi = min(total_rows, ((rank + 1) * units // world) * u)
    return slice(lo, hi)


def allreduce_bin_totals(bin_totals: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the int64 exponent-bin totals of the ranks' constants in place
    (integer addition: exact, in any order)."""
    assert bin_totals.dtype == torch.int64
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(bin_totals, op=dist.ReduceOp.SUM, group=group)
    return bin_totals


def quantize_nf4_dq_sharded(W_local: torch.Tensor, row_offset: int, total_rows: int, group=None, **kw):
    """Double-quantize rows [row_offset, row_offset + W_local.shape[0]) of a
    weight of total_rows rows whose other rows the other ranks of `group` hold
    (boundaries from shard_rows). Returns this rank's NF4Weight."""
    q, totals, ws = binding.qlora_quantize_nf4_dq_shard_begin(W_local, row_offset, total_rows, **kw)
    allreduce_bin_totals(totals, group)
    return binding.qlora_quantize_nf4_dq_shard_end(q, row_offset, total_rows, totals, ws,
                                                   stream=kw.get("stream"))
