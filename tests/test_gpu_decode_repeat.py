"""The decode forward is a fixed function of its inputs: calls repeated many times,
interleaved with other library calls and with allocations that leave garbage in
reused memory, must give bit-identical outputs. This catches ordering races in
the pipelined kernel (shared-memory stage reuse, split-tile tickets), which a
single parity check can miss."""
from __future__ import annotations

import random

import numpy as np
import pytest
import torch

from bit_nf4_quantized_absmax_b200 import binding as b
from bit_nf4_quantized_absmax_b200 import synthetic as syn
from tests.helpers import require_gpu

pytestmark = pytest.mark.gpu


def test_decode_repeated_calls_are_bit_identical():
    dev = require_gpu()
    cases = {}
    for shape in ((4096, 11008), (11008, 4096)):
        for M in (1, 4, 9, 16):
            inp = syn.make_linear(*shape, M, r=64, alpha=16.0, seed=0, workload="llama7b",
                                  layer=syn.LLAMA7B_SHAPES.index(shape))
            W, A, B, X = (t.to(dev) for t in (inp.W, inp.A, inp.B, inp.X))
            cases[(shape, M)] = (b.qlora_quantize_nf4_dq(W), X, A, B, inp.alpha)
    tr = syn.make_linear(256, 512, 200, r=24, alpha=16.0, seed=2, workload="test", dy_std=0.5)
    tW, tA, tB, tX, tdY = (t.to(dev) for t in (tr.W, tr.A, tr.B, tr.X, tr.dY))
    tq = b.qlora_quantize_nf4_dq(tW)

    def run(k):
        q, X, A, B, al = cases[k]
        Y, _ = b.qlora_linear_fwd(q, X, A, B, al)
        return Y.view(torch.int16).cpu().numpy()

    refs = {k: run(k) for k in cases}
    rng = random.Random(0)
    keys = list(cases)
    mismatches = []
    for it in range(320):
        p = rng.randrange(4)
        if p == 0:
            Y, T = b.qlora_linear_fwd(tq, tX, tA, tB, 16.0, T_save=True)
            b.qlora_linear_bwd(tq, tX, tA, tB, 16.0, tdY, T_saved=T)
        elif p == 1:
            junk = torch.empty(rng.randrange(1, 48) << 20, dtype=torch.uint8, device=dev)
            junk.fill_(rng.randrange(256))
            del junk
        elif p == 2:
            b.qlora_quantize_nf4_dq(tW)
        k = keys[rng.randrange(len(keys))]
        y = run(k)
        if not np.array_equal(y, refs[k]):
            mismatches.append((it, k, int((y != refs[k]).sum())))
    assert not mismatches, mismatches[:5]
    assert b.qlora_device_error() == 0
