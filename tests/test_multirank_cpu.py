"""Host logic of the multi-rank bench on CPU: world size 2 over gloo.

Each rank runs the same step on its own data (weak scaling, no data-path
collective); the only collectives are the barrier around the timed region and
the MAX of the per-rank times. The reference arm runs on rank 0 alone.
"""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    cpu = torch.device("cpu")
    bench.barrier(world)
    # each rank reports a different time; every rank must see the maximum
    got = bench.max_over_ranks(1.5 + rank, world, cpu)
    ref = bench.run_reference(type("A", (), {"steps": 1, "warmup": 0})(), rank, world) if rank == 1 else None
    bench.barrier(world)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"max": got, "ref_is_none": ref is None}, f)


def test_barrier_and_max_over_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    res = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(world)]
    assert [r_["max"] for r_ in res] == [2.5, 2.5]
    assert res[1]["ref_is_none"]


def test_max_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1, torch.device("cpu")) == 3.25


def test_ranks_draw_different_data():
    """Weak scaling: rank r seeds its workload with r, so ranks never share inputs."""
    from bit_nf4_quantized_absmax_b200 import synthetic as syn
    a = syn.make_linear(64, 128, 4, r=8, seed=0, workload="llama7b_train", layer=1)
    b = syn.make_linear(64, 128, 4, r=8, seed=1, workload="llama7b_train", layer=1)
    a2 = syn.make_linear(64, 128, 4, r=8, seed=0, workload="llama7b_train", layer=1)
    for k in ("W", "A", "B", "X", "dY"):
        assert not torch.equal(getattr(a, k), getattr(b, k))
        assert torch.equal(getattr(a, k), getattr(a2, k))


@pytest.mark.timeout(300)
def test_reference_arm_under_torchrun_prints_one_line():
    """`bench.py --impl reference` launched like the multi-GPU bench: rank 0
    alone runs the oracle and prints one JSON line; rank 1 exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="4")
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=280)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [json.loads(l_) for l_ in p.stdout.splitlines() if l_.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 1 and line["warmup"] == 3
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
