"""CPU-only checks of the C ABI: the library loads, exports every symbol the
header declares, and its host-side calls and argument checks behave as
documented. No kernel is launched here."""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from bit_nf4_quantized_absmax_b200 import binding as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora.h")


def _declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = b.load_library()
    declared = _declared_symbols()
    assert len(declared) >= 8
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(b.EXPORTED)


def test_header_is_plain_c():
    """The boundary header compiles as C99 and as C++ (no torch or CUDA types)."""
    import shutil
    import subprocess
    for cc, std, lang in (("gcc", "-std=c99", "c"), ("g++", "-std=c++17", "c++")):
        exe = shutil.which(cc)
        if exe is None:
            pytest.skip(f"{cc} not installed")
        res = subprocess.run([exe, std, "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-x", lang, HEADER],
                             capture_output=True, text=True)
        assert res.returncode == 0, res.stderr


def test_status_strings():
    assert b.qlora_status_string(0) == "QLORA_OK"
    assert b.qlora_status_string(5) == "QLORA_ERR_WORKSPACE"
    assert b.qlora_status_string(99) == "QLORA_ERR_UNKNOWN"


def test_codebook_equals_oracle_bits():
    """The library builds the codebook by Newton's method on erfc, the oracle by
    bisection: the fp32 bits agree."""
    lib_cb = b.qlora_nf4_codebook().numpy()
    assert np.array_equal(lib_cb.view(np.uint32), oracle.nf4_codebook().view(np.uint32))


def test_storage_bytes():
    assert b.qlora_nf4_storage_bytes(4096, 4096) == (8388608, 262144, 4096, 4)
    assert b.qlora_nf4_storage_bytes(3, 64 * 5) == (480, 15, 4, 4)
    sb = oracle.storage_bytes(11008, 4096)
    got = b.qlora_nf4_storage_bytes(11008, 4096)
    assert got == (sb["packed"], sb["absmax_q"], sb["dq_scale"], sb["mean"])
    with pytest.raises(b.QloraError) as e:
        b.qlora_nf4_storage_bytes(4, 100)
    assert e.value.status == 2


def _weight(rows=4, cols=128, **kw):
    fake = ctypes.c_void_p(1 << 20)  # aligned non-null dummies; nothing is launched
    w = b._Weight(fake.value, fake.value, fake.value, fake.value, rows, cols, 64, 256)
    for k, v in kw.items():
        setattr(w, k, v)
    return w


def test_argument_errors_return_before_launch():
    lib = b.load_library()
    n = ctypes.c_size_t(0)
    W = ctypes.c_void_p(1 << 20)
    # workspace size query launches nothing
    w = _weight()
    assert lib.qlora_quantize_nf4_dq(W, ctypes.byref(w), None, ctypes.byref(n), None) == 0
    assert n.value >= 4 * (4 * 128 // 64)
    # unsupported block sizes / columns
    assert lib.qlora_quantize_nf4_dq(W, ctypes.byref(_weight(blocksize=32)), None, ctypes.byref(n), None) == 2
    assert lib.qlora_quantize_nf4_dq(W, ctypes.byref(_weight(dq_blocksize=128)), None, ctypes.byref(n), None) == 2
    assert lib.qlora_quantize_nf4_dq(W, ctypes.byref(_weight(cols=100)), None, ctypes.byref(n), None) == 2
    # null pointers / negative sizes
    assert lib.qlora_quantize_nf4_dq(W, None, None, ctypes.byref(n), None) == 1
    assert lib.qlora_quantize_nf4_dq(W, ctypes.byref(_weight(rows=-1)), None, ctypes.byref(n), None) == 1
    assert lib.qlora_quantize_nf4_dq(W, ctypes.byref(_weight(packed=None)), None, ctypes.byref(n), None) == 1
    assert lib.qlora_quantize_nf4_dq(W, ctypes.byref(w), None, None, None) == 1
    # misaligned input or storage
    assert lib.qlora_quantize_nf4_dq(ctypes.c_void_p((1 << 20) + 2), ctypes.byref(w), None, ctypes.byref(n),
                                     None) == 3
    assert lib.qlora_quantize_nf4_dq(W, ctypes.byref(_weight(packed=(1 << 20) + 8)), None, ctypes.byref(n),
                                     None) == 3
    # workspace too small / misaligned
    small = ctypes.c_size_t(16)
    assert lib.qlora_quantize_nf4_dq(W, ctypes.byref(w), ctypes.c_void_p(1 << 20), ctypes.byref(small), None) == 5
    big = ctypes.c_size_t(1 << 30)
    assert lib.qlora_quantize_nf4_dq(W, ctypes.byref(w), ctypes.c_void_p((1 << 20) + 16), ctypes.byref(big),
                                     None) == 3
    # dequant: null output, misaligned output
    assert lib.qlora_dequantize_nf4_dq(ctypes.byref(w), None, None) == 1
    assert lib.qlora_dequantize_nf4_dq(ctypes.byref(w), ctypes.c_void_p((1 << 20) + 2), None) == 3
    # empty weight: nothing to do
    assert lib.qlora_dequantize_nf4_dq(ctypes.byref(_weight(rows=0)), None, None) == 0
    code = ctypes.c_int32(0)
    assert lib.qlora_device_error(None, None) == 1


def test_merge_argument_errors_return_before_launch():
    lib = b.load_library()
    w = _weight()
    fake = 1 << 20
    out = ctypes.c_void_p(fake)
    ok = b._Adapter(fake, fake, 16, 16.0, 1.0)
    arr = (b._Adapter * 9)(*([ok] * 9))
    assert lib.qlora_merge_lora(None, arr, 1, out, None) == 1                       # no weight
    assert lib.qlora_merge_lora(ctypes.byref(w), None, 1, out, None) == 1           # no adapter array
    assert lib.qlora_merge_lora(ctypes.byref(w), arr, -1, out, None) == 1           # negative count
    assert lib.qlora_merge_lora(ctypes.byref(w), arr, 9, out, None) == 2            # more than 8 adapters
    for bad, code in ((b._Adapter(fake, fake, 12, 16.0, 1.0), 2), (b._Adapter(fake, fake, 512, 16.0, 1.0), 2),
                      (b._Adapter(None, fake, 16, 16.0, 1.0), 1), (b._Adapter(fake + 8, fake, 16, 16.0, 1.0), 3)):
        one = (b._Adapter * 1)(bad)
        assert lib.qlora_merge_lora(ctypes.byref(w), one, 1, out, None) == code
    assert lib.qlora_merge_lora(ctypes.byref(w), arr, 1, None, None) == 1            # no output
    assert lib.qlora_merge_lora(ctypes.byref(w), arr, 1, ctypes.c_void_p(fake + 2), None) == 3  # misaligned output
    assert lib.qlora_merge_lora(ctypes.byref(_weight(rows=0)), arr, 1, None, None) == 0  # empty weight


def _single(rows=4, cols=128, **kw):
    fake = 1 << 20  # aligned non-null dummies; nothing is launched
    w = b._Weight(fake, None, None, None, rows, cols, 64, 0, fake)
    for k, v in kw.items():
        setattr(w, k, v)
    return w


def test_single_level_storage_bytes():
    assert b.qlora_nf4_single_storage_bytes(4096, 4096) == (8388608, 1048576)
    sb = oracle.storage_bytes(11008, 4096, double_quant=False)
    assert b.qlora_nf4_single_storage_bytes(11008, 4096) == (sb["packed"], sb["absmax"])
    assert sb["bits_per_param"] == 4.5  # 4-bit codes plus one fp32 constant per 64 weights
    with pytest.raises(b.QloraError) as e:
        b.qlora_nf4_single_storage_bytes(4, 100)
    assert e.value.status == 2


def test_single_level_argument_errors_return_before_launch():
    lib = b.load_library()
    W = ctypes.c_void_p(1 << 20)
    n = ctypes.c_size_t(0)
    fake = 1 << 20
    # each quantizer accepts only its own storage kind
    assert lib.qlora_quantize_nf4(W, ctypes.byref(_weight()), None) == 2
    assert lib.qlora_quantize_nf4_dq(W, ctypes.byref(_single()), None, ctypes.byref(n), None) == 2
    assert lib.qlora_quantize_nf4_dq_noalloc(W, ctypes.byref(_single()), None) == 2
    # null or misaligned single-level storage, input or output
    assert lib.qlora_quantize_nf4(W, ctypes.byref(_single(absmax=None)), None) == 1
    assert lib.qlora_quantize_nf4(W, ctypes.byref(_single(packed=None)), None) == 1
    assert lib.qlora_quantize_nf4(W, ctypes.byref(_single(absmax=fake + 2)), None) == 3
    assert lib.qlora_quantize_nf4(W, ctypes.byref(_single(packed=fake + 8)), None) == 3
    assert lib.qlora_quantize_nf4(None, ctypes.byref(_single()), None) == 1
    assert lib.qlora_quantize_nf4(ctypes.c_void_p(fake + 2), ctypes.byref(_single()), None) == 3
    assert lib.qlora_quantize_nf4(W, None, None) == 1
    assert lib.qlora_quantize_nf4(W, ctypes.byref(_single(cols=100)), None) == 2
    assert lib.qlora_quantize_nf4(W, ctypes.byref(_single(blocksize=32)), None) == 2
    assert lib.qlora_quantize_nf4(W, ctypes.byref(_single(rows=0)), None) == 0  # nothing to do
    # the dequantizers take either kind; other dq_blocksize values are unsupported
    for fn in (lib.qlora_dequantize_nf4, lib.qlora_dequantize_nf4_dq):
        assert fn(ctypes.byref(_single(absmax=None)), ctypes.c_void_p(fake), None) == 1
        assert fn(ctypes.byref(_single()), None, None) == 1
        assert fn(ctypes.byref(_single()), ctypes.c_void_p(fake + 2), None) == 3
        assert fn(ctypes.byref(_single(dq_blocksize=128)), ctypes.c_void_p(fake), None) == 2
        assert fn(ctypes.byref(_single(rows=0)), None, None) == 0
    # the linear layer and the merge check the single-level storage the same way
    assert lib.qlora_linear_fwd(ctypes.byref(_single(absmax=None)), W, 1, W, W, 16, 16.0, W, None, None,
                                ctypes.byref(n), None) == 1
    assert lib.qlora_linear_fwd(ctypes.byref(_single()), W, 1, W, W, 12, 16.0, W, None, None,
                                ctypes.byref(n), None) == 2
    assert lib.qlora_linear_fwd(ctypes.byref(_single()), W, 1, W, W, 16, 16.0, W, None, None,
                                ctypes.byref(n), None) == 0 and n.value > 0  # size query
    ok = (b._Adapter * 1)(b._Adapter(fake, fake, 16, 16.0, 1.0))
    assert lib.qlora_merge_lora(ctypes.byref(_single(absmax=fake + 1)), ok, 1, ctypes.c_void_p(fake), None) == 3


def test_optimizer_argument_errors_return_before_launch():
    lib = b.load_library()
    fake = 1 << 20
    P = ctypes.c_void_p(fake)
    args = dict(lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, wd=0.0, step=1)

    def call(p=P, pb=None, g=P, m=P, v=P, n=1024, **kw):
        a = {**args, **kw}
        return lib.qlora_adamw_step(p, pb, g, m, v, n, a["lr"], a["b1"], a["b2"], a["eps"], a["wd"], a["step"], None)

    assert call(n=0) == 0                         # nothing to do
    assert call(n=-1) == 1
    assert call(step=0) == 1
    assert call(b1=1.0) == 1 and call(b2=-0.1) == 1 and call(eps=0.0) == 1 and call(lr=-1.0) == 1
    assert call(wd=-0.5) == 1
    assert call(g=None) == 1 and call(m=None) == 1 and call(p=None) == 1
    assert call(p=ctypes.c_void_p(fake + 4)) == 3  # fp32 buffers need 16-byte alignment
    assert call(g=ctypes.c_void_p(fake + 2)) == 3  # bf16 buffers need 8-byte alignment
    assert call(pb=ctypes.c_void_p(fake + 2)) == 3
    out = ctypes.c_void_p(123)
    assert lib.qlora_paged_alloc(0, 0, ctypes.byref(out)) == 1 and out.value in (None, 0, 123)
    assert lib.qlora_paged_alloc(1024, 0, None) == 1
    assert lib.qlora_paged_free(None) == 0
    assert lib.qlora_paged_prefetch(None, 16, 0, None) == 1
