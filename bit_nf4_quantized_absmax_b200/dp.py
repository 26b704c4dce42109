"""Data-parallel QLoRA training step across ranks (one process per GPU).

Every rank holds the same frozen weight (its own NF4 copy: quantization is a
fixed function of the weight, so the copies are bit-identical without any
exchange) and the same LoRA parameters, and processes its own shard of the
tokens. The forward needs nothing from other ranks and dX stays with the rank
that owns the tokens; the only exchange is the sum of the LoRA gradients dA
and dB over ranks. Each rank's backward (qlora_linear_bwd_dp) writes them in
fp32 into one flat buffer and records an event as soon as they are complete,
before its dX kernels; a side stream waits on that event, sums the buffer over
the ranks with one all-reduce (NCCL over NVLink on GPUs) while dX is computed,
and rounds the sums once to bf16 in the library (qlora_round_bf16), as a
single-GPU backward rounds its own. This module holds no arithmetic of its own:
the kernels run through `binding`, the sum is the collective.

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


def _distributed(group) -> bool:
    return dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1


def flat_grads(r: int, K: int, N: int, device=None, dtype=torch.float32) -> tuple:
    """One flat buffer of r*K + N*r values and its two views (dA [r, K], dB [N, r]),
    in the layout qlora_linear_bwd_dp writes."""
    buf = torch.empty(r * K + N * r, dtype=dtype, device=device)
    return buf, buf[:r * K].view(r, K), buf[r * K:].view(N, r)


def allreduce_grads(buf: torch.Tensor, group=None) -> torch.Tensor:
    """Sum a flat gradient buffer over the ranks of `group`, in place (the
    exchange of the data-parallel step; any torch.distributed backend)."""
    if _distributed(group):
        dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
    return buf


_SIDE = {}


def _side_stream(device: torch.device) -> torch.cuda.Stream:
    """One side stream per device for the gradient exchange."""
    key = device.index if device.index is not None else torch.cuda.current_device()
    if key not in _SIDE:
        _SIDE[key] = torch.cuda.Stream(device=device)
    return _SIDE[key]


def dp_linear_fwd(q, X_local: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float, **kw):
    """Forward of this rank's token shard (no exchange). Returns (Y_local, T_local)."""
    return binding.qlora_linear_fwd(q, X_local, A, B, alpha, T_save=True, **kw)


def dp_linear_bwd(q, X_local: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float, dY_local: torch.Tensor,
                  T_local: torch.Tensor | None = None, need_dX: bool = True, group=None, stream=None,
                  workspace: torch.Tensor | None = None):
    """Backward of this rank's token shard. The fp32 LoRA gradients are summed over
    the ranks on a side stream while this rank's dX is computed, then rounded once
    to bf16 by the library. Returns (dX_local or None, dA, dB); dA and dB are bf16
    and equal on every rank. On return, `stream` (default: the current stream) is
    ordered after the exchange, so every output is ready for its next kernel."""
    dev = X_local.device
    main = torch.cuda.current_stream(dev) if stream is None else stream
    r, K, N = A.shape[0], q.cols, q.rows
    with torch.cuda.stream(main):
        grads, _, _ = flat_grads(r, K, N, device=dev)
        out, dA, dB = flat_grads(r, K, N, device=dev, dtype=torch.bfloat16)
    ready = torch.cuda.Event()
    dX = binding.qlora_linear_bwd_dp(q, X_local, A, B, alpha, dY_local, grads, T_saved=T_local, need_dX=need_dX,
                                     grads_ready=ready, workspace=workspace, stream=main)
    side = _side_stream(dev)
    side.wait_event(ready)
    with torch.cuda.stream(side):
        allreduce_grads(grads, group)        # the collective is ordered after `side`, and `side` after it
        binding.qlora_round_bf16(grads, out, stream=side)
    main.wait_stream(side)                   # dX overlapped the exchange; the outputs are ready on `main`
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
    if _distributed(group):
        dist.all_reduce(bin_totals, op=dist.ReduceOp.SUM, group=group)
    return bin_totals


def quantize_nf4_dq_sharded(W_local: torch.Tensor, row_offset: int, total_rows: int, group=None, stream=None,
                            **kw):
    """Double-quantize rows [row_offset, row_offset + W_local.shape[0]) of a
    weight of total_rows rows whose other rows the other ranks of `group` hold
    (boundaries from shard_rows). The library calls and the exchange run in
    order on `stream` (default: the current stream). Returns this rank's NF4Weight."""
    st = torch.cuda.current_stream(W_local.device) if stream is None else stream
    q, totals, ws = binding.qlora_quantize_nf4_dq_shard_begin(W_local, row_offset, total_rows, stream=st, **kw)
    with torch.cuda.stream(st):
        allreduce_bin_totals(totals, group)
    return binding.qlora_quantize_nf4_dq_shard_end(q, row_offset, total_rows, totals, ws, stream=st)
