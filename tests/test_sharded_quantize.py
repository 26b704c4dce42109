"""Double quantization of one weight split by rows over several ranks.

The shards exchange only the exact sum of their block constants (256 integer
exponent-bin totals); their outputs must equal the whole weight's, bit for bit.

- CPU: the argument checks of the two C-ABI calls (nothing is launched), and two
  gloo ranks that each take level 1 of their rows from the oracle, form the
  bin totals, sum them with the module's all-reduce and finish level 2 with
  the resulting mean; the concatenation equals the oracle's whole-weight result.
- GPU: the library's shard calls, on one device, against its whole-weight call
  and the oracle.
"""
from __future__ import annotations

import ctypes
import datetime
import os
import socket
import sys
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from bit_nf4_quantized_absmax_b200 import binding as b  # noqa: E402
from bit_nf4_quantized_absmax_b200 import dp  # noqa: E402
from bit_nf4_quantized_absmax_b200 import synthetic as syn  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _weight_case(rows=300, cols=768, seed=31):
    return syn.make_linear(rows, cols, 4, r=16, alpha=16.0, seed=seed, workload="test").W


def _bin_totals(absmax: np.ndarray) -> np.ndarray:
    """The exchange format: each constant is sig * 2^(E - 134) (8-bit significand
    sig, E = max(exponent field, 1)); totals[E] = sum of sig over the bin."""
    u = np.asarray(absmax, dtype=np.float32).view(np.uint32).astype(np.int64)
    assert np.all(u & 0xFFFF == 0) and np.all(u >> 31 == 0)  # non-negative bf16 values
    e = (u >> 23) & 0xFF
    mant7 = (u >> 16) & 0x7F
    sig = np.where(e > 0, mant7 | 0x80, mant7)
    return np.bincount(np.maximum(e, 1), weights=sig, minlength=256).astype(np.int64)


def _mean_from_totals(totals: np.ndarray, nblk: int) -> np.float32:
    """mu = fp32(fp64(S) / nblk) with S = sum_E totals[E] 2^(E - 134), exactly."""
    S = sum(Fraction(int(t)) * Fraction(2) ** (E - 134) for E, t in enumerate(totals) if t)
    return np.float32(np.float64(float(S)) / np.float64(nblk))


# ---- CPU: argument checks -------------------------------------------------

def _weight(rows=128, cols=128, **kw):
    fake = ctypes.c_void_p(1 << 20)  # aligned non-null dummies; nothing is launched
    w = b._Weight(fake.value, fake.value, fake.value, fake.value, rows, cols, 64, 256)
    for k, v in kw.items():
        setattr(w, k, v)
    return w


def test_shard_argument_errors_return_before_launch():
    lib = b.load_library()
    W = ctypes.c_void_p(1 << 20)
    tot = ctypes.c_void_p(1 << 21)
    n = ctypes.c_size_t(0)
    begin, end = lib.qlora_quantize_nf4_dq_shard_begin, lib.qlora_quantize_nf4_dq_shard_end
    # cols = 128: a 256-constant group spans 128 rows
    assert begin(W, ctypes.byref(_weight()), 0, 300, tot, None, ctypes.byref(n), None) == 0
    assert n.value >= 4 * 128 * 128 // 64
    assert begin(W, ctypes.byref(_weight(rows=44)), 256, 300, tot, None, ctypes.byref(n), None) == 0  # ragged last
    assert begin(W, ctypes.byref(_weight(rows=0)), 128, 300, tot, None, ctypes.byref(n), None) == 0  # empty shard
    # shard not on a group boundary, or a non-last shard that does not end on one
    assert begin(W, ctypes.byref(_weight()), 4, 300, tot, None, ctypes.byref(n), None) == 1
    assert begin(W, ctypes.byref(_weight(rows=100)), 0, 300, tot, None, ctypes.byref(n), None) == 1
    # shard beyond the weight, negative sizes
    assert begin(W, ctypes.byref(_weight()), 256, 300, tot, None, ctypes.byref(n), None) == 1
    assert begin(W, ctypes.byref(_weight()), -128, 300, tot, None, ctypes.byref(n), None) == 1
    assert begin(W, ctypes.byref(_weight(rows=-1)), 0, 300, tot, None, ctypes.byref(n), None) == 1
    assert begin(W, None, 0, 300, tot, None, ctypes.byref(n), None) == 1
    assert begin(W, ctypes.byref(_weight()), 0, 300, tot, None, None, None) == 1
    # storage kind and sizes
    assert begin(W, ctypes.byref(_weight(dq_blocksize=0)), 0, 300, tot, None, ctypes.byref(n), None) == 2
    assert begin(W, ctypes.byref(_weight(cols=100)), 0, 300, tot, None, ctypes.byref(n), None) == 2
    assert begin(W, ctypes.byref(_weight(cols=1 << 30)), 0, 1 << 27, tot, None, ctypes.byref(n), None) == 2
    # workspace, totals and input checks (with a workspace given)
    ws = ctypes.c_void_p(1 << 22)
    small = ctypes.c_size_t(16)
    big = ctypes.c_size_t(1 << 30)
    assert begin(W, ctypes.byref(_weight()), 0, 300, tot, ws, ctypes.byref(small), None) == 5
    assert begin(W, ctypes.byref(_weight()), 0, 300, tot, ctypes.c_void_p((1 << 22) + 16), ctypes.byref(big),
                 None) == 3
    assert begin(W, ctypes.byref(_weight()), 0, 300, None, ws, ctypes.byref(big), None) == 1
    assert begin(W, ctypes.byref(_weight()), 0, 300, ctypes.c_void_p((1 << 21) + 4), ws, ctypes.byref(big),
                 None) == 3
    assert begin(None, ctypes.byref(_weight()), 0, 300, tot, ws, ctypes.byref(big), None) == 1
    assert begin(ctypes.c_void_p((1 << 20) + 2), ctypes.byref(_weight()), 0, 300, tot, ws, ctypes.byref(big),
                 None) == 3
    assert begin(W, ctypes.byref(_weight(packed=(1 << 20) + 8)), 0, 300, tot, ws, ctypes.byref(big), None) == 3
    # end: same shard rules, then workspace and totals
    assert end(ctypes.byref(_weight()), 4, 300, tot, ws, 1 << 30, None) == 1
    assert end(ctypes.byref(_weight(rows=0)), 128, 300, None, None, 0, None) == 0  # empty shard: nothing to do
    assert end(ctypes.byref(_weight()), 0, 300, tot, None, 1 << 30, None) == 1
    assert end(ctypes.byref(_weight()), 0, 300, tot, ws, 16, None) == 5
    assert end(ctypes.byref(_weight()), 0, 300, tot, ctypes.c_void_p((1 << 22) + 16), 1 << 30, None) == 3
    assert end(ctypes.byref(_weight()), 0, 300, None, ws, 1 << 30, None) == 1
    assert end(ctypes.byref(_weight()), 0, 300, ctypes.c_void_p((1 << 21) + 4), ws, 1 << 30, None) == 3


def test_shard_rows_are_group_aligned_and_cover_every_row():
    for cols in (64, 128, 768, 4096, 11008, 16384, 22016):
        u = dp.group_aligned_rows(cols)
        assert (u * cols) % 16384 == 0 and all((v * cols) % 16384 for v in range(1, u))
        for total in (0, 1, 63, 64, 300, 1000, 11008):
            for world in (1, 2, 3, 8):
                spans = [dp.shard_rows(total, cols, r, world) for r in range(world)]
                assert spans[0].start == 0 and spans[-1].stop == total
                for a, c in zip(spans, spans[1:]):
                    assert a.stop == c.start
                for s in spans:
                    assert (s.start * cols) % 16384 == 0
                    assert s.stop == total or ((s.stop - s.start) * cols) % 16384 == 0


def test_bin_totals_give_the_exact_mean():
    """The integer exchange format reproduces the oracle's correctly rounded
    mean (math.fsum), including subnormal and widely spread constants."""
    rng = np.random.default_rng(5)
    for m in (np.abs(rng.standard_normal(5000)).astype(np.float32) * 0.05,
              np.float32([2.0 ** -130, 2.0 ** -126, 1.5 * 2.0 ** 100, 3.0, 0.0, 2.0 ** -133]),
              np.float32(2.0) ** rng.integers(-140, 120, 3000).astype(np.float32)):
        m = (m.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)  # bf16-valued, as absmax of bf16 weights
        got = _mean_from_totals(_bin_totals(m), m.size)
        assert got.view(np.uint32) == oracle.dq_mean(m).view(np.uint32)


# ---- CPU: two gloo ranks ----------------------------------------------------

def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from tests.helpers import bf16_to_f32_np
    W = bf16_to_f32_np(_weight_case())
    rows, cols = W.shape
    sl = dp.shard_rows(rows, cols, rank, world)
    codes, absmax = oracle.quantize_nf4(W[sl], oracle.nf4_codebook())
    totals = torch.from_numpy(_bin_totals(absmax))
    dp.allreduce_bin_totals(totals)
    mu = _mean_from_totals(totals.numpy(), rows * cols // 64)
    q, scale, mu_used = oracle.double_quantize(absmax, mean=mu)
    dist.barrier()
    dist.destroy_process_group()
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), packed=oracle.pack_codes(codes), q=q, scale=scale,
             mu=np.float32(mu_used), lo=sl.start, hi=sl.stop)


def test_sharded_dq_over_two_ranks_equals_whole_weight(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    from tests.helpers import bf16_to_f32_np
    ref = oracle.quantize_nf4_dq(bf16_to_f32_np(_weight_case()))
    parts = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    assert int(parts[0]["lo"]) == 0 and int(parts[0]["hi"]) == int(parts[1]["lo"]) > 0
    assert int(parts[1]["hi"]) == ref.rows
    for p in parts:
        assert p["mu"].view(np.uint32) == np.float32(ref.mean).view(np.uint32)
    assert np.array_equal(np.concatenate([p["packed"] for p in parts]), ref.packed)
    assert np.array_equal(np.concatenate([p["q"] for p in parts]), ref.absmax_q)
    assert np.array_equal(np.concatenate([p["scale"] for p in parts]).view(np.uint32), ref.dq_scale.view(np.uint32))


# ---- GPU: the library's shard calls ------------------------------------------

def _shard_on_gpu(W, world):
    rows, cols = W.shape
    spans = [dp.shard_rows(rows, cols, r, world) for r in range(world)]
    begun = [b.qlora_quantize_nf4_dq_shard_begin(W[s], s.start, rows) for s in spans]
    total = begun[0][1].clone()
    for _, t, _ in begun[1:]:
        total += t
    qs = [b.qlora_quantize_nf4_dq_shard_end(q, s.start, rows, total, ws) for s, (q, _, ws) in zip(spans, begun)]
    return spans, qs


@pytest.mark.gpu
@pytest.mark.parametrize("rows,cols,world", [(300, 768, 2), (300, 768, 3), (64, 768, 3), (11008, 4096, 4)])
def test_gpu_sharded_matches_whole_weight(rows, cols, world):
    from tests.helpers import bf16_bits_np, require_gpu
    dev = require_gpu()
    W = _weight_case(rows, cols, seed=rows + world).to(dev).contiguous()
    whole = b.qlora_quantize_nf4_dq(W)
    Wd = b.qlora_dequantize_nf4_dq(whole)
    spans, qs = _shard_on_gpu(W, world)
    Wd_parts = [b.qlora_dequantize_nf4_dq(q) for q in qs if q.rows > 0]
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    for q in qs:
        if q.rows > 0:
            assert torch.equal(q.mean.view(torch.int32), whole.mean.view(torch.int32))
    assert torch.equal(torch.cat([q.packed for q in qs]), whole.packed)
    assert torch.equal(torch.cat([q.absmax_q for q in qs]), whole.absmax_q)
    assert torch.equal(torch.cat([q.dq_scale for q in qs]).view(torch.int32), whole.dq_scale.view(torch.int32))
    assert np.array_equal(bf16_bits_np(torch.cat(Wd_parts)), bf16_bits_np(Wd))
    if rows * cols <= 300 * 768:  # and the oracle, at the small size
        ref = oracle.quantize_nf4_dq(W.float().cpu().numpy())
        assert np.array_equal(torch.cat([q.absmax_q for q in qs]).cpu().numpy(), ref.absmax_q)
        assert np.array_equal(torch.cat([q.packed for q in qs]).cpu().numpy(), ref.packed)
    # through the module, one rank without a process group: the whole weight
    one = dp.quantize_nf4_dq_sharded(W, 0, rows)
    torch.cuda.synchronize()
    assert torch.equal(one.absmax_q, whole.absmax_q) and torch.equal(one.packed, whole.packed)
