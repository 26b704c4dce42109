"""The allocation-free quantize entry point (qlora_quantize_nf4_dq_noalloc).

Some callers cannot allocate device memory or hand the library a workspace:
serving runtimes that plan all device memory at start-up, or hosts where
cudaMalloc's implicit device synchronization is not acceptable. For them the
library offers a quantize call whose scratch is a fixed array inside the
library. This test calls it through the C ABI twice in a row and checks that
each call gives exactly the outputs of the regular entry point, and that a
weight too large for the fixed scratch is rejected before any launch.

The file is named so that pytest collects it last.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from bit_nf4_quantized_absmax_b200 import binding as b
from bit_nf4_quantized_absmax_b200 import synthetic as syn
from tests.helpers import require_gpu

pytestmark = pytest.mark.gpu


def _same(q1: b.NF4Weight, q2: b.NF4Weight):
    assert torch.equal(q1.packed, q2.packed)
    assert torch.equal(q1.absmax_q, q2.absmax_q)
    assert torch.equal(q1.dq_scale.view(torch.int32), q2.dq_scale.view(torch.int32))
    assert torch.equal(q1.mean.view(torch.int32), q2.mean.view(torch.int32))


def test_noalloc_matches_regular_entry_point_twice():
    dev = require_gpu()
    lib = b.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # first a large weight, then a smaller one with a different distribution, so
    # leftovers of the first call in the shared scratch would show up
    cases = [syn.normal_bf16((4096, 11008), 0.02, 0, "test", 301),
             syn.student_t_bf16((1000, 4160), 4, 0.02, 0, "test", 302)]
    for W_cpu in cases:
        W = W_cpu.to(dev)
        ref = b.qlora_quantize_nf4_dq(W)
        out = b.NF4Weight.empty(W.shape[0], W.shape[1], dev)
        for t in (out.packed, out.absmax_q, out.dq_scale, out.mean):
            t.fill_(0x5A if t.dtype in (torch.uint8, torch.int8) else 7.0)
        qc = out.as_c()
        st = lib.qlora_quantize_nf4_dq_noalloc(ctypes.c_void_p(W.data_ptr()), ctypes.byref(qc), stream)
        assert st == 0, b.qlora_status_string(st)
        torch.cuda.synchronize()
        _same(out, ref)
    assert b.qlora_device_error() == 0


def test_noalloc_rejects_weights_beyond_its_scratch():
    require_gpu()
    lib = b.load_library()
    # 2^22 blocks of 64 is the limit; one row more is rejected before launching
    fake = 1 << 20
    w = b._Weight(fake, fake, fake, fake, (1 << 22) // 64 + 1, 64 * 64, 64, 256)
    assert lib.qlora_quantize_nf4_dq_noalloc(ctypes.c_void_p(fake), ctypes.byref(w), None) == 2
