"""Thin ctypes binding of the C ABI in include/qlora.h.

Argument marshalling only: torch tensors supply device memory and the current
stream; every step of the computation runs in the library's CUDA kernels. The
functions keep the C names. Loading fails loudly when the shared library has
not been built; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqlora_b200.so")

QLORA_OK = 0
STATUS_NAMES = {0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARG", 2: "QLORA_ERR_UNSUPPORTED", 3: "QLORA_ERR_ALIGNMENT",
                4: "QLORA_ERR_CUDA", 5: "QLORA_ERR_WORKSPACE", 6: "QLORA_ERR_DEVICE"}

EXPORTED = ("qlora_status_string", "qlora_nf4_codebook", "qlora_nf4_storage_bytes", "qlora_nf4_single_storage_bytes",
            "qlora_quantize_nf4", "qlora_quantize_nf4_dq", "qlora_quantize_nf4_dq_noalloc",
            "qlora_quantize_nf4_dq_shard_begin", "qlora_quantize_nf4_dq_shard_end", "qlora_dequantize_nf4",
            "qlora_dequantize_nf4_dq", "qlora_linear_fwd", "qlora_linear_bwd", "qlora_linear_bwd_f32",
            "qlora_linear_bwd_dp", "qlora_round_bf16", "qlora_merge_lora", "qlora_codebook", "qlora_quantize_4bit",
            "qlora_dequantize_4bit", "qlora_linear_fwd_multi", "qlora_pack_adapters",
            "qlora_paged_alloc", "qlora_paged_free", "qlora_paged_prefetch", "qlora_adamw_step",
            "qlora_device_error")


class QloraError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


class _Weight(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("absmax_q", ctypes.c_void_p), ("dq_scale", ctypes.c_void_p),
                ("mean", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("blocksize", ctypes.c_int32), ("dq_blocksize", ctypes.c_int32), ("absmax", ctypes.c_void_p)]


_lib = None


class _Adapter(ctypes.Structure):
    _fields_ = [("A", ctypes.c_void_p), ("B", ctypes.c_void_p), ("r", ctypes.c_int32), ("alpha", ctypes.c_float),
                ("weight", ctypes.c_float)]


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libqlora_b200.so (once). Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m bit_nf4_quantized_absmax_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    wp = ctypes.POINTER(_Weight)
    szp = ctypes.POINTER(ctypes.c_size_t)
    lib.qlora_status_string.restype = ctypes.c_char_p
    lib.qlora_status_string.argtypes = [ctypes.c_int]
    lib.qlora_nf4_codebook.argtypes = [ctypes.POINTER(ctypes.c_float)]
    lib.qlora_nf4_storage_bytes.argtypes = [i64, i64, ctypes.POINTER(sz)]
    lib.qlora_nf4_single_storage_bytes.argtypes = [i64, i64, ctypes.POINTER(sz)]
    lib.qlora_quantize_nf4.argtypes = [vp, wp, vp]
    lib.qlora_dequantize_nf4.argtypes = [wp, vp, vp]
    lib.qlora_quantize_nf4_dq.argtypes = [vp, wp, vp, szp, vp]
    lib.qlora_quantize_nf4_dq_noalloc.argtypes = [vp, wp, vp]
    lib.qlora_quantize_nf4_dq_shard_begin.argtypes = [vp, wp, i64, i64, vp, vp, szp, vp]
    lib.qlora_quantize_nf4_dq_shard_end.argtypes = [wp, i64, i64, vp, vp, sz, vp]
    lib.qlora_dequantize_nf4_dq.argtypes = [wp, vp, vp]
    lib.qlora_linear_fwd.argtypes = [wp, vp, i64, vp, vp, i32, f32, vp, vp, vp, szp, vp]
    lib.qlora_linear_bwd.argtypes = [wp, vp, i64, vp, vp, i32, f32, vp, vp, vp, vp, vp, vp, szp, vp]
    lib.qlora_linear_bwd_f32.argtypes = [wp, vp, i64, vp, vp, i32, f32, vp, vp, vp, vp, vp, vp, szp, vp]
    lib.qlora_linear_bwd_dp.argtypes = [wp, vp, i64, vp, vp, i32, f32, vp, vp, vp, vp, vp, vp, szp, vp]
    lib.qlora_round_bf16.argtypes = [vp, vp, i64, vp]
    lib.qlora_codebook.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_float)]
    lib.qlora_quantize_4bit.argtypes = [vp, wp, ctypes.c_int, vp, szp, vp]
    lib.qlora_dequantize_4bit.argtypes = [wp, ctypes.c_int, vp, vp]
    lib.qlora_linear_fwd_multi.argtypes = [wp, vp, i64, vp, vp, i32, vp, vp, vp, szp, vp]
    lib.qlora_pack_adapters.argtypes = [ctypes.POINTER(_Adapter), i32, i64, i64, vp, vp, vp, vp]
    lib.qlora_merge_lora.argtypes = [wp, ctypes.POINTER(_Adapter), i32, vp, vp]
    lib.qlora_device_error.argtypes = [ctypes.POINTER(ctypes.c_int32), vp]
    lib.qlora_paged_alloc.argtypes = [sz, i32, ctypes.POINTER(vp)]
    lib.qlora_paged_free.argtypes = [vp]
    lib.qlora_paged_prefetch.argtypes = [vp, sz, i32, vp]
    lib.qlora_adamw_step.argtypes = [vp, vp, vp, vp, vp, i64, f32, f32, f32, f32, f32, i64, vp]
    for name in EXPORTED:
        getattr(lib, name).restype = ctypes.c_int if name != "qlora_status_string" else ctypes.c_char_p
    _lib = lib
    return lib


def _check(status: int, what: str):
    if status != QLORA_OK:
        raise QloraError(status, what)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


@dataclass
class NF4Weight:
    """Device storage of one quantized frozen weight [rows, cols]."""
    packed: torch.Tensor     # uint8 [rows*cols/2]
    absmax_q: torch.Tensor   # int8 [nblk]
    dq_scale: torch.Tensor   # float32 [ngrp]
    mean: torch.Tensor       # float32 [1]
    rows: int
    cols: int

    def as_c(self) -> _Weight:
        return _Weight(self.packed.data_ptr(), self.absmax_q.data_ptr(), self.dq_scale.data_ptr(),
                       self.mean.data_ptr(), self.rows, self.cols, 64, 256)

    @staticmethod
    def empty(rows: int, cols: int, device="cuda") -> "NF4Weight":
        sizes = qlora_nf4_storage_bytes(rows, cols)
        return NF4Weight(torch.empty(sizes[0], dtype=torch.uint8, device=device),
                         torch.empty(sizes[1], dtype=torch.int8, device=device),
                         torch.empty(sizes[2] // 4, dtype=torch.float32, device=device),
                         torch.empty(1, dtype=torch.float32, device=device), rows, cols)


@dataclass
class SingleNF4Weight:
    """Single-level storage of one quantized weight [rows, cols]: codes and the
    fp32 block constants (no double quantization)."""
    packed: torch.Tensor     # uint8 [rows*cols/2]
    absmax: torch.Tensor     # float32 [nblk]
    rows: int
    cols: int

    def as_c(self) -> _Weight:
        return _Weight(self.packed.data_ptr(), None, None, None, self.rows, self.cols, 64, 0,
                       self.absmax.data_ptr())

    @staticmethod
    def empty(rows: int, cols: int, device="cuda") -> "SingleNF4Weight":
        sizes = qlora_nf4_single_storage_bytes(rows, cols)
        return SingleNF4Weight(torch.empty(sizes[0], dtype=torch.uint8, device=device),
                               torch.empty(sizes[1] // 4, dtype=torch.float32, device=device), rows, cols)


def qlora_status_string(status: int) -> str:
    return load_library().qlora_status_string(status).decode()


def qlora_nf4_codebook() -> torch.Tensor:
    out = (ctypes.c_float * 16)()
    _check(load_library().qlora_nf4_codebook(out), "qlora_nf4_codebook")
    return torch.tensor(list(out), dtype=torch.float32)


DTYPE_NF4, DTYPE_FP4 = 0, 1


def qlora_codebook(dtype: int = DTYPE_NF4) -> torch.Tensor:
    """The 16 values of a 4-bit data type (DTYPE_NF4 or DTYPE_FP4), ascending."""
    out = (ctypes.c_float * 16)()
    _check(load_library().qlora_codebook(dtype, out), "qlora_codebook")
    return torch.tensor(list(out), dtype=torch.float32)


def qlora_quantize_4bit(W: torch.Tensor, dtype: int, double_quant: bool = True, out=None,
                        workspace: torch.Tensor | None = None, stream=None):
    """Quantize with the codebook of `dtype`; double-quantized (NF4Weight) or
    single-level (SingleNF4Weight) storage."""
    assert W.dtype == torch.bfloat16 and W.dim() == 2 and W.is_contiguous()
    lib = load_library()
    if out is None:
        out = (NF4Weight if double_quant else SingleNF4Weight).empty(W.shape[0], W.shape[1], W.device)
    qc = out.as_c()
    st = _stream(stream)
    ws, nbytes = _workspace(lambda p, n: lib.qlora_quantize_4bit(_ptr(W), ctypes.byref(qc), dtype, p, n, st),
                            workspace, W.device)
    _check(lib.qlora_quantize_4bit(_ptr(W), ctypes.byref(qc), dtype, _ptr(ws), ctypes.byref(nbytes), st),
           "qlora_quantize_4bit")
    return out


def qlora_dequantize_4bit(q, dtype: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Dequantize either storage kind with the codebook of `dtype` to bf16."""
    if out is None:
        out = torch.empty(q.rows, q.cols, dtype=torch.bfloat16, device=q.packed.device)
    qc = q.as_c()
    _check(load_library().qlora_dequantize_4bit(ctypes.byref(qc), dtype, _ptr(out), _stream(stream)),
           "qlora_dequantize_4bit")
    return out


def qlora_nf4_storage_bytes(rows: int, cols: int) -> tuple:
    out = (ctypes.c_size_t * 4)()
    _check(load_library().qlora_nf4_storage_bytes(rows, cols, out), "qlora_nf4_storage_bytes")
    return tuple(int(x) for x in out)


def qlora_nf4_single_storage_bytes(rows: int, cols: int) -> tuple:
    out = (ctypes.c_size_t * 2)()
    _check(load_library().qlora_nf4_single_storage_bytes(rows, cols, out), "qlora_nf4_single_storage_bytes")
    return tuple(int(x) for x in out)


def _workspace(query, workspace: torch.Tensor | None, device) -> tuple:
    """Run the size query; return (workspace tensor, ctypes size)."""
    need = ctypes.c_size_t(0)
    _check(query(None, ctypes.byref(need)), "workspace query")
    if workspace is None or workspace.numel() < need.value:
        workspace = torch.empty(max(need.value, 256), dtype=torch.uint8, device=device)
    return workspace, ctypes.c_size_t(workspace.numel())


def qlora_quantize_nf4_dq(W: torch.Tensor, out: NF4Weight | None = None, workspace: torch.Tensor | None = None,
                          stream=None) -> NF4Weight:
    assert W.dtype == torch.bfloat16 and W.dim() == 2 and W.is_contiguous()
    lib = load_library()
    q = out or NF4Weight.empty(W.shape[0], W.shape[1], W.device)
    qc = q.as_c()
    st = _stream(stream)
    ws, nbytes = _workspace(lambda p, n: lib.qlora_quantize_nf4_dq(_ptr(W), ctypes.byref(qc), p, n, st), workspace,
                            W.device)
    _check(lib.qlora_quantize_nf4_dq(_ptr(W), ctypes.byref(qc), _ptr(ws), ctypes.byref(nbytes), st),
           "qlora_quantize_nf4_dq")
    return q


def qlora_quantize_nf4(W: torch.Tensor, out: SingleNF4Weight | None = None, stream=None) -> SingleNF4Weight:
    """Single-level quantization (codes and fp32 block constants)."""
    assert W.dtype == torch.bfloat16 and W.dim() == 2 and W.is_contiguous()
    q = out or SingleNF4Weight.empty(W.shape[0], W.shape[1], W.device)
    qc = q.as_c()
    _check(load_library().qlora_quantize_nf4(_ptr(W), ctypes.byref(qc), _stream(stream)), "qlora_quantize_nf4")
    return q


def qlora_quantize_nf4_dq_noalloc(W: torch.Tensor, out: NF4Weight, stream=None) -> NF4Weight:
    """Quantize into `out` without any device allocation by the library (its
    scratch is a fixed array inside the library; see include/qlora.h)."""
    assert W.dtype == torch.bfloat16 and W.dim() == 2 and W.is_contiguous()
    qc = out.as_c()
    _check(load_library().qlora_quantize_nf4_dq_noalloc(_ptr(W), ctypes.byref(qc), _stream(stream)),
           "qlora_quantize_nf4_dq_noalloc")
    return out


def qlora_quantize_nf4_dq_shard_begin(W_shard: torch.Tensor, row_offset: int, total_rows: int,
                                      out: NF4Weight | None = None, bin_totals: torch.Tensor | None = None,
                                      workspace: torch.Tensor | None = None, stream=None) -> tuple:
    """Level 1 of rows [row_offset, row_offset + rows) of a weight with total_rows
    rows that several callers quantize in row shards. Returns (q, bin_totals,
    workspace): q holds the shard's codes, bin_totals (int64 [256], device) the
    exact sum of its block constants by exponent bin, to be summed over all
    shards before qlora_quantize_nf4_dq_shard_end, and the workspace the shard's
    fp32 constants, to be kept until then."""
    assert W_shard.dtype == torch.bfloat16 and W_shard.dim() == 2 and W_shard.is_contiguous()
    lib = load_library()
    dev = W_shard.device
    q = out or NF4Weight.empty(W_shard.shape[0], W_shard.shape[1], dev)
    if bin_totals is None:
        bin_totals = torch.empty(256, dtype=torch.int64, device=dev)
    assert bin_totals.dtype == torch.int64 and bin_totals.numel() == 256 and bin_totals.is_contiguous()
    qc = q.as_c()
    st = _stream(stream)
    ws, nbytes = _workspace(lambda p, n: lib.qlora_quantize_nf4_dq_shard_begin(
        _ptr(W_shard), ctypes.byref(qc), row_offset, total_rows, _ptr(bin_totals), p, n, st), workspace, dev)
    _check(lib.qlora_quantize_nf4_dq_shard_begin(_ptr(W_shard), ctypes.byref(qc), row_offset, total_rows,
                                                 _ptr(bin_totals), _ptr(ws), ctypes.byref(nbytes), st),
           "qlora_quantize_nf4_dq_shard_begin")
    return q, bin_totals, ws


def qlora_quantize_nf4_dq_shard_end(q: NF4Weight, row_offset: int, total_rows: int, bin_totals: torch.Tensor,
                                    workspace: torch.Tensor, stream=None) -> NF4Weight:
    """Level 2 of a row shard once bin_totals holds the sum over all shards: the
    mean of all constants of the weight, then this shard's int8 codes and group
    scales (bit-identical to the same rows of a whole-weight quantization)."""
    assert bin_totals.dtype == torch.int64 and bin_totals.numel() == 256 and bin_totals.is_contiguous()
    qc = q.as_c()
    _check(load_library().qlora_quantize_nf4_dq_shard_end(ctypes.byref(qc), row_offset, total_rows,
                                                          _ptr(bin_totals), _ptr(workspace), workspace.numel(),
                                                          _stream(stream)),
           "qlora_quantize_nf4_dq_shard_end")
    return q


def qlora_dequantize_nf4(q: NF4Weight | SingleNF4Weight, out: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """Dequantize either storage kind to bf16."""
    lib = load_library()
    if out is None:
        out = torch.empty(q.rows, q.cols, dtype=torch.bfloat16, device=q.packed.device)
    qc = q.as_c()
    _check(lib.qlora_dequantize_nf4(ctypes.byref(qc), _ptr(out), _stream(stream)), "qlora_dequantize_nf4")
    return out


def qlora_dequantize_nf4_dq(q: NF4Weight | SingleNF4Weight, out: torch.Tensor | None = None,
                            stream=None) -> torch.Tensor:
    lib = load_library()
    if out is None:
        out = torch.empty(q.rows, q.cols, dtype=torch.bfloat16, device=q.packed.device)
    qc = q.as_c()
    _check(lib.qlora_dequantize_nf4_dq(ctypes.byref(qc), _ptr(out), _stream(stream)), "qlora_dequantize_nf4_dq")
    return out


def qlora_linear_fwd(q: NF4Weight | SingleNF4Weight, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float,
                     Y: torch.Tensor | None = None, T_save: torch.Tensor | bool | None = None,
                     workspace: torch.Tensor | None = None, stream=None):
    """Returns (Y, T) with T = X A^T in fp32 when T_save is True or a tensor, else (Y, None)."""
    lib = load_library()
    M, r = X.shape[0], A.shape[0]
    dev = X.device
    if Y is None:
        Y = torch.empty(M, q.rows, dtype=torch.bfloat16, device=dev)
    if T_save is True:
        T_save = torch.empty(M, r, dtype=torch.float32, device=dev)
    elif T_save is False:
        T_save = None
    qc = q.as_c()
    st = _stream(stream)
    args = lambda p, n: lib.qlora_linear_fwd(ctypes.byref(qc), _ptr(X), M, _ptr(A), _ptr(B), r, float(alpha),
                                             _ptr(Y), _ptr(T_save), p, n, st)
    ws, nbytes = _workspace(args, workspace, dev)
    _check(args(_ptr(ws), ctypes.byref(nbytes)), "qlora_linear_fwd")
    return Y, T_save


def qlora_linear_bwd(q: NF4Weight | SingleNF4Weight, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float,
                     dY: torch.Tensor, T_saved: torch.Tensor | None = None, need_dX: bool = True,
                     dX: torch.Tensor | None = None, dA: torch.Tensor | None = None, dB: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, grads_fp32: bool = False, stream=None):
    """Returns (dX or None, dA, dB); dA and dB are fp32 with grads_fp32 (qlora_linear_bwd_f32), else bf16."""
    lib = load_library()
    M, r = X.shape[0], A.shape[0]
    dev = X.device
    gdt = torch.float32 if grads_fp32 else torch.bfloat16
    if need_dX and dX is None:
        dX = torch.empty(M, q.cols, dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty(r, q.cols, dtype=gdt, device=dev)
    if dB is None:
        dB = torch.empty(q.rows, r, dtype=gdt, device=dev)
    assert dA.dtype == gdt and dB.dtype == gdt
    qc = q.as_c()
    st = _stream(stream)
    fn = lib.qlora_linear_bwd_f32 if grads_fp32 else lib.qlora_linear_bwd
    args = lambda p, n: fn(ctypes.byref(qc), _ptr(X), M, _ptr(A), _ptr(B), r, float(alpha), _ptr(dY), _ptr(T_saved),
                           _ptr(dX if need_dX else None), _ptr(dA), _ptr(dB), p, n, st)
    ws, nbytes = _workspace(args, workspace, dev)
    _check(args(_ptr(ws), ctypes.byref(nbytes)), "qlora_linear_bwd_f32" if grads_fp32 else "qlora_linear_bwd")
    return (dX if need_dX else None), dA, dB


def qlora_linear_bwd_dp(q: NF4Weight | SingleNF4Weight, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                        alpha: float, dY: torch.Tensor, grads: torch.Tensor, T_saved: torch.Tensor | None = None,
                        need_dX: bool = True, dX: torch.Tensor | None = None, grads_ready=None,
                        workspace: torch.Tensor | None = None, stream=None):
    """Backward of one token shard with dA and dB in fp32 in one flat buffer
    `grads` [r*K + N*r] (dA first); `grads_ready` (a torch.cuda.Event or None) is
    recorded on the stream once `grads` is complete, before the dX kernels.
    Returns dX or None."""
    lib = load_library()
    M, r = X.shape[0], A.shape[0]
    dev = X.device
    assert grads.dtype == torch.float32 and grads.is_contiguous() and grads.numel() == r * q.cols + q.rows * r
    if need_dX and dX is None:
        dX = torch.empty(M, q.cols, dtype=torch.bfloat16, device=dev)
    ev = None
    if grads_ready is not None:
        grads_ready.record(torch.cuda.current_stream() if stream is None else stream)  # creates the CUDA event
        ev = ctypes.c_void_p(grads_ready.cuda_event)
    qc = q.as_c()
    st = _stream(stream)
    args = lambda p, n: lib.qlora_linear_bwd_dp(ctypes.byref(qc), _ptr(X), M, _ptr(A), _ptr(B), r, float(alpha),
                                                _ptr(dY), _ptr(T_saved), _ptr(dX if need_dX else None), _ptr(grads),
                                                ev, p, n, st)
    ws, nbytes = _workspace(args, workspace, dev)
    _check(args(_ptr(ws), ctypes.byref(nbytes)), "qlora_linear_bwd_dp")
    return dX if need_dX else None


def qlora_round_bf16(src: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """bf16_rn of an fp32 tensor, in the library's kernel."""
    assert src.dtype == torch.float32 and src.is_contiguous()
    if out is None:
        out = torch.empty(src.shape, dtype=torch.bfloat16, device=src.device)
    assert out.dtype == torch.bfloat16 and out.is_contiguous() and out.numel() == src.numel()
    _check(load_library().qlora_round_bf16(_ptr(src), _ptr(out), src.numel(), _stream(stream)), "qlora_round_bf16")
    return out


def qlora_pack_adapters(adapters, rows: int, cols: int, device=None, stream=None) -> tuple:
    """Concatenate adapters [(A [r, cols], B [rows, r], alpha, weight), ...] along
    the rank for qlora_linear_fwd_multi. Returns (A_cat, B_cat, col_scale)."""
    dev = device or adapters[0][0].device
    rt = sum(A.shape[0] for A, _, _, _ in adapters)
    A_cat = torch.empty(rt, cols, dtype=torch.bfloat16, device=dev)
    B_cat = torch.empty(rows, rt, dtype=torch.bfloat16, device=dev)
    col_scale = torch.empty(rt, dtype=torch.float32, device=dev)
    arr = (_Adapter * len(adapters))()
    for i, (A, B, alpha, weight) in enumerate(adapters):
        arr[i] = _Adapter(_ptr(A), _ptr(B), A.shape[0], float(alpha), float(weight))
    _check(load_library().qlora_pack_adapters(arr, len(adapters), rows, cols, _ptr(A_cat), _ptr(B_cat),
                                              _ptr(col_scale), _stream(stream)), "qlora_pack_adapters")
    return A_cat, B_cat, col_scale


def qlora_linear_fwd_multi(q, X: torch.Tensor, A_cat: torch.Tensor, B_cat: torch.Tensor, col_scale: torch.Tensor,
                           Y: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """Y = X W'^T + sum_a c_a (X A_a^T) B_a^T from the packed adapters."""
    lib = load_library()
    M, rt = X.shape[0], A_cat.shape[0]
    if Y is None:
        Y = torch.empty(M, q.rows, dtype=torch.bfloat16, device=X.device)
    qc = q.as_c()
    st = _stream(stream)
    args = lambda p, n: lib.qlora_linear_fwd_multi(ctypes.byref(qc), _ptr(X), M, _ptr(A_cat), _ptr(B_cat), rt,
                                                   _ptr(col_scale), _ptr(Y), p, n, st)
    ws, nbytes = _workspace(args, workspace, X.device)
    _check(args(_ptr(ws), ctypes.byref(nbytes)), "qlora_linear_fwd_multi")
    return Y


def qlora_merge_lora(q: NF4Weight | SingleNF4Weight, adapters, out: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Merged bf16 weight [rows, cols] from the NF4 base and a sequence of
    adapters (A [r, cols], B [rows, r], alpha, weight); see include/qlora.h."""
    lib = load_library()
    if out is None:
        out = torch.empty(q.rows, q.cols, dtype=torch.bfloat16, device=q.packed.device)
    arr = (_Adapter * max(1, len(adapters)))()
    for i, (A, B, alpha, weight) in enumerate(adapters):
        arr[i] = _Adapter(_ptr(A), _ptr(B), A.shape[0], float(alpha), float(weight))
    qc = q.as_c()
    _check(lib.qlora_merge_lora(ctypes.byref(qc), arr, len(adapters), _ptr(out), _stream(stream)),
           "qlora_merge_lora")
    return out


def qlora_device_error(stream=None) -> int:
    code = ctypes.c_int32(0)
    _check(load_library().qlora_device_error(ctypes.byref(code), _stream(stream)), "qlora_device_error")
    return int(code.value)


class PagedBuffer:
    """Paged (managed) device memory from qlora_paged_alloc, freed with the object
    or by free(). tensor(dtype, n) views it as a torch tensor; keep the buffer
    alive while such views are in use."""

    def __init__(self, nbytes: int, device: int | None = None):
        dev = torch.cuda.current_device() if device is None else device
        ptr = ctypes.c_void_p()
        _check(load_library().qlora_paged_alloc(nbytes, dev, ctypes.byref(ptr)), "qlora_paged_alloc")
        self.ptr, self.nbytes, self.device = ptr.value, nbytes, dev

    def tensor(self, dtype: torch.dtype, n: int) -> torch.Tensor:
        itemsize = torch.empty(0, dtype=dtype).element_size()
        assert n * itemsize <= self.nbytes
        typestr = {torch.float32: "<f4", torch.bfloat16: "<i2", torch.uint8: "|u1"}[dtype]
        owner = self

        class _View:
            __cuda_array_interface__ = {"shape": (n,), "typestr": typestr, "data": (owner.ptr, False),
                                        "version": 3, "strides": None}
        t = torch.as_tensor(_View(), device=f"cuda:{self.device}")
        return t.view(dtype) if dtype == torch.bfloat16 else t

    def prefetch(self, device: int, stream=None):
        """Move the buffer to GPU `device`, or to host memory with device == -1."""
        _check(load_library().qlora_paged_prefetch(ctypes.c_void_p(self.ptr), self.nbytes, device, _stream(stream)),
               "qlora_paged_prefetch")

    def free(self):
        if self.ptr:
            _check(load_library().qlora_paged_free(ctypes.c_void_p(self.ptr)), "qlora_paged_free")
            self.ptr = None

    def __del__(self):
        try:
            if self.ptr:
                torch.cuda.synchronize(self.device)
                self.free()
        except Exception:  # noqa: BLE001 -- interpreter shutdown
            pass


def qlora_adamw_step(param: torch.Tensor, grad: torch.Tensor, exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor,
                     step: int, lr: float = 1e-3, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
                     weight_decay: float = 0.0, param_bf16: torch.Tensor | None = None, stream=None):
    """One AdamW step over flat fp32 parameters with bf16 gradients (see include/qlora.h)."""
    assert param.dtype == torch.float32 and exp_avg.dtype == torch.float32 and exp_avg_sq.dtype == torch.float32
    assert grad.dtype == torch.bfloat16
    n = param.numel()
    assert grad.numel() == n and exp_avg.numel() == n and exp_avg_sq.numel() == n
    _check(load_library().qlora_adamw_step(_ptr(param), _ptr(param_bf16), _ptr(grad), _ptr(exp_avg),
                                           _ptr(exp_avg_sq), n, float(lr), float(beta1), float(beta2), float(eps),
                                           float(weight_decay), int(step), _stream(stream)), "qlora_adamw_step")
