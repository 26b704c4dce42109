"""Benchmark of the QLoRA NF4 hot path on B200.

One step = one pass of the whole hot path over the Llama-7B linear shapes
(4096x4096, 11008x4096, 4096x11008), r = 64, alpha = 16, seeded synthetic data:
  quantize + double-quantize W, dequantize W, decode forward at M = 1, 4, 16,
  training forward at M = 4096 and training backward (dX, dA, dB) at M = 4096.
The headline value is training TFLOP/s: the useful flops of the M = 4096
forward + backward (2MNK + 2Mr(K+N) and 2MNK + 4Mr(K+N)) divided by the time
of the whole step. Per-part times, decode weight GB/s and the roofline of the
dominant kernel are reported beside it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torch.distributed.run, one rank per GPU, as data-parallel
training (weak scaling): every rank runs the step on its own 4096 training
tokens per linear and the LoRA gradients of the backward are summed over the
ranks in fp32 by one NCCL all-reduce per linear, on a side stream that overlaps
the rank's dX GEMM; the time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_nf4_quantized_absmax_b200 import binding as qb  # noqa: E402
from bit_nf4_quantized_absmax_b200 import synthetic as syn  # noqa: E402

METRIC = "fused NF4+LoRA linear TFLOP/s (M=4096) and weight GB/s (M=1..16) vs roofline"
R, ALPHA, M_TRAIN, M_DECODE = 64, 16.0, 4096, (1, 4, 16)
SHAPES = syn.LLAMA7B_SHAPES

# DRAM traffic of the roofline call (qlora_linear_fwd, M=4096, 11008x4096: dequant,
# LoRA-down GEMM, finish, 2-CTA GEMM) summed from one ncu capture of
# `bench.py --profile-case` (dram__bytes_read.sum + dram__bytes_write.sum per
# launch, one pass). Valid only for the kernel sources it was taken on.
ROOFLINE_SHAPE = (11008, 4096)
TRAFFIC_RECORD = {"fingerprint": "6808c8a4a1587ff7", "bytes": 303.8e6}
TRAFFIC_SOURCES = ("common.cuh", "nf4_lut.cuh", "dequant.cu", "gemm_tc.cu", "lora_misc.cu", "api.cu")


def source_fingerprint():
    import hashlib
    h = hashlib.sha1()
    for f in TRAFFIC_SOURCES:
        h.update(open(os.path.join(ROOT, "bit_nf4_quantized_absmax_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


# device spin (clock cycles) queued before a call timed with its own event pair
HOST_AHEAD_CYCLES = 200_000

# kernels each C-ABI call launches on these shapes (see the launchers in csrc/)
LAUNCHES = {"quantize": 3, "dequantize": 1, "decode_fwd": 2, "train_fwd": 4, "train_bwd": 9}


def train_flops(N, K, M=M_TRAIN, r=R):
    fwd = 2 * M * N * K + 2 * M * r * (K + N)
    bwd = 2 * M * N * K + 4 * M * r * (K + N)
    return fwd, bwd


def decode_bytes(N, K, M, r=R, single=False):
    return weight_bytes(N, K, single) + 2 * r * (K + N) + 2 * M * (K + N)


def quant_bytes(N, K, single=False):
    # read bf16 W, write codes + int8 constants + scales (single-level: + fp32 constants)
    return (2.5625 if single else 2.516) * N * K


def weight_bytes(N, K, single=False):
    return (0.5625 if single else 0.515869) * N * K


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"qlora_clocks_{os.getpid()}.csv")
        self.t_begin = self.t_end = None

    def start(self):
        """Start sampling (before the warm-up, so samples exist when timing starts)."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu=timestamp,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def mark_begin(self):
        self.t_begin = time.time()

    def mark_end(self):
        self.t_end = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        import datetime as _dt
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = _dt.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            if self.t_begin is not None and not (self.t_begin - 0.25 <= ts <= self.t_end + 0.25):
                continue
            f = f[1:]
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------
# our arm

class Workload:
    """Device-resident inputs, outputs and workspaces of one step. With dp=True
    (N > 1 ranks) every rank's backward is the data-parallel one: dA and dB in
    fp32 in one flat buffer, summed over the ranks by an NCCL all-reduce on a side
    stream while the rank's dX GEMM runs, then rounded once to bf16."""

    def __init__(self, dev, seed, dp=False):
        self.dev = dev
        self.dp = dp
        self.side = torch.cuda.Stream(device=dev) if dp else None
        self.lin = []
        for li, (N, K) in enumerate(SHAPES):
            inp = syn.make_linear(N, K, M_TRAIN, r=R, alpha=ALPHA, seed=seed, workload="llama7b_train", layer=li)
            d = {k: getattr(inp, k).to(dev).contiguous() for k in ("W", "A", "B", "X", "dY")}
            d["N"], d["K"] = N, K
            d["Xdec"] = {M: d["X"][:M].contiguous() for M in M_DECODE}
            d["q"] = qb.NF4Weight.empty(N, K, dev)
            d["Wd"] = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
            d["Ydec"] = {M: torch.empty(M, N, dtype=torch.bfloat16, device=dev) for M in M_DECODE}
            d["Y"] = torch.empty(M_TRAIN, N, dtype=torch.bfloat16, device=dev)
            d["T"] = torch.empty(M_TRAIN, R, dtype=torch.float32, device=dev)
            d["dX"] = torch.empty(M_TRAIN, K, dtype=torch.bfloat16, device=dev)
            d["dA"] = torch.empty(R, K, dtype=torch.bfloat16, device=dev)
            d["dB"] = torch.empty(N, R, dtype=torch.bfloat16, device=dev)
            if dp:  # flat fp32 sums and their bf16 rounding: dA [R, K] then dB [N, R]
                d["grads"] = torch.empty(R * K + N * R, dtype=torch.float32, device=dev)
                d["grads_bf16"] = torch.empty(R * K + N * R, dtype=torch.bfloat16, device=dev)
                d["ev"] = torch.cuda.Event()
                d["ev"].record()  # creates the CUDA event
            self.lin.append(d)
        self.ws = torch.empty(self._ws_bytes(), dtype=torch.uint8, device=dev)

    def _ws_bytes(self):
        import ctypes
        lib = qb.load_library()
        need = 0
        for d in self.lin:
            for fn in (self._q_call, self._fwd_call, self._bwd_call):
                n = ctypes.c_size_t(0)
                fn(lib, d, None, n, None, M_TRAIN)
                need = max(need, n.value)
            n = ctypes.c_size_t(0)
            self._fwd_call(lib, d, None, n, None, 16)
            need = max(need, n.value)
        return need

    # raw C-ABI calls (workspace == None: size query)
    @staticmethod
    def _q_call(lib, d, ws, n, st, M):
        import ctypes
        qc = d["q"].as_c()
        return lib.qlora_quantize_nf4_dq(qb._ptr(d["W"]), ctypes.byref(qc), ws, ctypes.byref(n), st)

    @staticmethod
    def _fwd_call(lib, d, ws, n, st, M):
        import ctypes
        qc = d["q"].as_c()
        X = d["X"] if M == M_TRAIN else d["Xdec"][M]
        Y = d["Y"] if M == M_TRAIN else d["Ydec"][M]
        T = d["T"] if M == M_TRAIN else None
        return lib.qlora_linear_fwd(ctypes.byref(qc), qb._ptr(X), M, qb._ptr(d["A"]), qb._ptr(d["B"]), R, ALPHA,
                                    qb._ptr(Y), qb._ptr(T), ws, ctypes.byref(n), st)

    @staticmethod
    def _bwd_call(lib, d, ws, n, st, M):
        import ctypes
        qc = d["q"].as_c()
        return lib.qlora_linear_bwd(ctypes.byref(qc), qb._ptr(d["X"]), M, qb._ptr(d["A"]), qb._ptr(d["B"]), R,
                                    ALPHA, qb._ptr(d["dY"]), qb._ptr(d["T"]), qb._ptr(d["dX"]), qb._ptr(d["dA"]),
                                    qb._ptr(d["dB"]), ws, ctypes.byref(n), st)

    @staticmethod
    def _bwd_dp_call(lib, d, ws, n, st, M):
        import ctypes
        qc = d["q"].as_c()
        return lib.qlora_linear_bwd_dp(ctypes.byref(qc), qb._ptr(d["X"]), M, qb._ptr(d["A"]), qb._ptr(d["B"]), R,
                                       ALPHA, qb._ptr(d["dY"]), qb._ptr(d["T"]), qb._ptr(d["dX"]),
                                       qb._ptr(d["grads"]), ctypes.c_void_p(d["ev"].cuda_event), ws, ctypes.byref(n),
                                       st)

    def _exchange(self, lib, d):
        """Sum the rank's flat fp32 LoRA gradients over all ranks on the side stream
        (after the backward's event, overlapping its dX GEMM) and round them to bf16."""
        import ctypes
        main = torch.cuda.current_stream()
        self.side.wait_event(d["ev"])
        with torch.cuda.stream(self.side):
            torch.distributed.all_reduce(d["grads"])
            rc = lib.qlora_round_bf16(qb._ptr(d["grads"]), qb._ptr(d["grads_bf16"]), d["grads"].numel(),
                                      ctypes.c_void_p(self.side.cuda_stream))
        main.wait_stream(self.side)
        return rc

    def step(self, ev=None, only=None, lins=None):
        """One pass of the hot path. ev: optional dict part -> list of (start, end)
        events, recorded for the parts named in `only` (all parts if None).
        lins: the linears to run (all if None)."""
        import ctypes
        lib = qb.load_library()
        st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        ws = ctypes.c_void_p(self.ws.data_ptr())
        n = ctypes.c_size_t(self.ws.numel())

        def rec(part, fn):
            if ev is not None and (only is None or part in only):
                # the device first spins for ~0.1 ms, so that the host has queued the
                # call's launches before the device reaches the start event: the two
                # events then bracket device execution, not host launch gaps
                torch.cuda._sleep(HOST_AHEAD_CYCLES)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                rc = fn()
                b.record()
                ev.setdefault(part, []).append((a, b))
            else:
                rc = fn()
            if rc != 0:
                raise qb.QloraError(rc, part)

        for li, d in enumerate(self.lin):
            if lins is not None and li not in lins:
                continue
            rec(f"quantize/{li}", lambda: self._q_call(lib, d, ws, n, st, 0))
            qc = d["q"].as_c()
            rec(f"dequantize/{li}", lambda: lib.qlora_dequantize_nf4_dq(ctypes.byref(qc), qb._ptr(d["Wd"]), st))
            for M in M_DECODE:
                rec(f"decode{M}/{li}", lambda: self._fwd_call(lib, d, ws, n, st, M))
            rec(f"train_fwd/{li}", lambda: self._fwd_call(lib, d, ws, n, st, M_TRAIN))
            if self.dp:
                rec(f"train_bwd/{li}", lambda: self._bwd_dp_call(lib, d, ws, n, st, M_TRAIN))
                rec(f"exchange/{li}", lambda: self._exchange(lib, d))
            else:
                rec(f"train_bwd/{li}", lambda: self._bwd_call(lib, d, ws, n, st, M_TRAIN))

    def launches_per_step(self):
        per = LAUNCHES["quantize"] + LAUNCHES["dequantize"] + len(M_DECODE) * LAUNCHES["decode_fwd"] + \
            LAUNCHES["train_fwd"] + LAUNCHES["train_bwd"] + (1 if self.dp else 0)  # + the bf16 rounding
        return per * len(self.lin)


class E2EStreams:
    """A copy stream and per-linear events for the end-to-end step."""

    def __init__(self, n):
        self.copy = torch.cuda.Stream()
        self.copied = [torch.cuda.Event() for _ in range(n)]   # inputs of linear i on the device
        self.done = [torch.cuda.Event() for _ in range(n)]     # linear i's compute and read-back issued
        for e in self.done:
            e.record()


def e2e_step(work: Workload, host, streams: E2EStreams, start=None):
    """The same step through the public API with host buffers: pinned H2D copies
    of each linear's inputs on a copy stream (linear i + 1's while linear i
    computes; a linear's buffers are refilled only after its previous use), the
    step's calls for that linear once its copy has landed, and a D2H read of its
    results."""
    main = torch.cuda.current_stream()
    h2d = 0
    with torch.cuda.stream(streams.copy):
        if start is not None:  # nothing of a timed step runs before its start event
            streams.copy.wait_event(start)
        for li, (d, h) in enumerate(zip(work.lin, host)):
            streams.copy.wait_event(streams.done[li])
            for k in ("W", "A", "B", "X", "dY"):
                d[k].copy_(h[k], non_blocking=True)
                h2d += h[k].numel() * h[k].element_size()
            for M in M_DECODE:
                d["Xdec"][M].copy_(d["X"][:M], non_blocking=True)
            streams.copied[li].record(streams.copy)
    d2h = 0
    for li, (d, h) in enumerate(zip(work.lin, host)):
        main.wait_event(streams.copied[li])
        work.step(lins={li})
        for k in (("grads_bf16",) if work.dp else ("dA", "dB")):  # the LoRA gradients of the step
            h["out_" + k].copy_(d[k], non_blocking=True)
            d2h += d[k].numel() * d[k].element_size()
        for M in M_DECODE:
            h[f"out_Y{M}"].copy_(d["Ydec"][M], non_blocking=True)
            d2h += d["Ydec"][M].numel() * 2
        streams.done[li].record(main)
    return h2d, d2h


def breakdown(work, dev, reps=24):
    """Mean time per call (us) of every part of the step, L2-cold inputs."""
    import ctypes
    lib = qb.load_library()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ws = ctypes.c_void_p(work.ws.data_ptr())
    n = ctypes.c_size_t(work.ws.numel())
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 128 << 20)
    out = {}

    def timed(part, calls):
        for c in calls[:3]:
            c()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(reps):
            rc = calls[i % len(calls)]()
            if rc != 0:
                raise qb.QloraError(rc, part)
        b.record()
        torch.cuda.synchronize()
        out[part] = 1e3 * a.elapsed_time(b) / reps

    for li, d in enumerate(work.lin):
        N, K = d["N"], d["K"]
        nw = max(2, math.ceil(2 * l2 / (2 * N * K)))
        nq = max(2, math.ceil(2 * l2 / (0.515869 * N * K)))
        Ws = [d["W"]] + [d["W"].clone() for _ in range(nw - 1)]
        Wds = [d["Wd"]] + [torch.empty_like(d["Wd"]) for _ in range(nw - 1)]
        qs = [d["q"]]
        for _ in range(nq - 1):
            qn = qb.NF4Weight.empty(N, K, dev)
            for name in ("packed", "absmax_q", "dq_scale", "mean"):
                getattr(qn, name).copy_(getattr(d["q"], name))
            qs.append(qn)
        qcs = [q.as_c() for q in qs]

        def q_call(i, li=li):
            return lib.qlora_quantize_nf4_dq(qb._ptr(Ws[i % nw]), ctypes.byref(qcs[i % nq]), ws, ctypes.byref(n), st)

        timed(f"quantize/{li}", [lambda i=i: q_call(i) for i in range(max(nw, nq))])
        timed(f"dequantize/{li}", [lambda i=i: lib.qlora_dequantize_nf4_dq(ctypes.byref(qcs[i % nq]),
                                                                            qb._ptr(Wds[i % nw]), st)
                                   for i in range(max(nw, nq))])
        for M in M_DECODE:
            X, Y = d["Xdec"][M], d["Ydec"][M]
            timed(f"decode{M}/{li}", [lambda qc=qc, X=X, Y=Y, M=M: lib.qlora_linear_fwd(
                ctypes.byref(qc), qb._ptr(X), M, qb._ptr(d["A"]), qb._ptr(d["B"]), R, ALPHA, qb._ptr(Y), None, ws,
                ctypes.byref(n), st) for qc in qcs])
        timed(f"train_fwd/{li}", [lambda d=d: work._fwd_call(lib, d, ws, n, st, M_TRAIN)])
        timed(f"train_bwd/{li}", [lambda d=d: work._bwd_call(lib, d, ws, n, st, M_TRAIN)])
        if li == 1:  # single-level storage (fp32 block constants), outside the step: one shape
            ns = max(2, math.ceil(2 * l2 / (0.5625 * N * K)))
            ss = [qb.qlora_quantize_nf4(d["W"]) for _ in range(ns)]
            scs = [q.as_c() for q in ss]
            timed(f"quantize_single/{li}", [lambda i=i: lib.qlora_quantize_nf4(
                qb._ptr(Ws[i % nw]), ctypes.byref(scs[i % ns]), st) for i in range(max(nw, ns))])
            timed(f"dequantize_single/{li}", [lambda i=i: lib.qlora_dequantize_nf4(
                ctypes.byref(scs[i % ns]), qb._ptr(Wds[i % nw]), st) for i in range(max(nw, ns))])
            for M in M_DECODE:
                X, Y = d["Xdec"][M], d["Ydec"][M]
                timed(f"decode{M}_single/{li}", [lambda qc=qc, X=X, Y=Y, M=M: lib.qlora_linear_fwd(
                    ctypes.byref(qc), qb._ptr(X), M, qb._ptr(d["A"]), qb._ptr(d["B"]), R, ALPHA, qb._ptr(Y), None,
                    ws, ctypes.byref(n), st) for qc in scs])
            del ss, scs
        del Ws, Wds, qs, qcs
        torch.cuda.empty_cache()
    return out


def capture_step_graph(work, say):
    """One step of the hot path captured into a CUDA graph, or None."""
    try:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            work.step()  # settle lazy per-kernel attributes outside the capture
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            work.step()
        torch.cuda.synchronize()
        return g
    except Exception as e:  # noqa: BLE001
        say(f"graph capture failed ({e}); timing stream launches only")
        return None


def merge_measure(work, dev, reps=10):
    """Adapter merge (outside the step): one r = 64 adapter
    merged into the 11008x4096 base, W' + s B A in fp64, back to back."""
    import ctypes
    lib = qb.load_library()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    d = work.lin[SHAPES.index(ROOFLINE_SHAPE)]
    N, K = d["N"], d["K"]
    out = d["Wd"]
    arr = (qb._Adapter * 1)(qb._Adapter(qb._ptr(d["A"]), qb._ptr(d["B"]), R, ALPHA, 1.0))
    qc = d["q"].as_c()
    call = lambda: lib.qlora_merge_lora(ctypes.byref(qc), arr, 1, qb._ptr(out), st)  # noqa: E731
    for _ in range(2):
        call()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        if call() != 0:
            raise qb.QloraError(1, "qlora_merge_lora")
    b.record()
    torch.cuda.synchronize()
    us = 1e3 * a.elapsed_time(b) / reps
    flops = 2.0 * R * N * K
    # no fp64 peak was measured on this machine, so no roofline fraction is given
    return {"shape": f"{N}x{K}", "r": R, "us": round(us, 1), "fp64_TFLOP_s": round(flops / us / 1e6, 2),
            "peak": None, "peak_note": "fp64 peak not measured here (nominal B200 fp64 is about 40 TFLOP/s)"}


def adamw_measure(dev, peaks, n=1 << 26, reps=10):
    """Paged AdamW step (outside the step) over n flat fp32 parameters with bf16
    gradients: once with device-resident state, once with the moments in paged
    (managed) memory prefetched to the GPU. 28 bytes per parameter: p, m, v read
    and written (24), the bf16 gradient read and the bf16 copy of p written (4)."""
    import ctypes
    lib = qb.load_library()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = torch.randn(n, device=dev) * 0.02
    g = (torch.randn(n, device=dev) * 1e-2).to(torch.bfloat16)
    pb = torch.empty(n, dtype=torch.bfloat16, device=dev)
    m, v = torch.zeros(n, device=dev), torch.zeros(n, device=dev)
    bm, bv = qb.PagedBuffer(4 * n), qb.PagedBuffer(4 * n)
    mp, vp = bm.tensor(torch.float32, n), bv.tensor(torch.float32, n)
    mp.zero_()
    vp.zero_()
    bm.prefetch(bm.device)
    bv.prefetch(bv.device)
    out = {"n": n, "bytes_per_param": 28}
    for name, (mm, vv) in (("device", (m, v)), ("paged", (mp, vp))):
        def call(t):
            return lib.qlora_adamw_step(qb._ptr(p), qb._ptr(pb), qb._ptr(g), qb._ptr(mm), qb._ptr(vv), n, 1e-4, 0.9,
                                        0.999, 1e-8, 0.0, t, st)
        for t in range(1, 3):
            call(t)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for t in range(3, 3 + reps):
            if call(t) != 0:
                raise qb.QloraError(1, "qlora_adamw_step")
        b.record()
        torch.cuda.synchronize()
        us = 1e3 * a.elapsed_time(b) / reps
        gbs = 28.0 * n / us / 1e3
        out[name] = {"us": round(us, 1), "GB_s": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 4)}
    del mp, vp
    bm.free()
    bv.free()
    return out


def _timed_calls(calls, reps):
    """Mean time per call (us) of `reps` calls cycling through `calls`, back to back."""
    for c in calls[:3]:
        c()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(reps):
        rc = calls[i % len(calls)]()
        if rc not in (0, None):
            raise qb.QloraError(rc, "timed call")
    b.record()
    torch.cuda.synchronize()
    return 1e3 * a.elapsed_time(b) / reps


def measure_llama65b(dev, peaks, reps=12):
    """Llama-65B linear shapes (8192x8192, 22016x8192, 8192x22016) with Student-t(4)
    weights scaled to std 0.02: quantize + DQ and dequant GB/s, decode (M = 1)
    weight GB/s, and forward + backward TFLOP/s at M = 2048 tokens. Each call back
    to back, rotating copies of its inputs beyond twice the L2 where they fit in it."""
    import ctypes
    lib = qb.load_library()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 128 << 20)
    M = 2048
    out, fl_tot, us_tot = {}, 0.0, 0.0
    for li, (N, K) in enumerate(syn.LLAMA65B_SHAPES):
        base = 16 * li
        W = syn.student_t_bf16_device((N, K), 4, 0.02, 0, "llama65b", base + 0, device=dev)
        A = syn.normal_bf16_device((R, K), 0.02, 0, "llama65b", base + 1, device=dev)
        B = syn.normal_bf16_device((N, R), 0.02, 0, "llama65b", base + 2, device=dev)
        X = syn.normal_bf16_device((M, K), 1.0, 0, "llama65b", base + 3, device=dev)
        dY = syn.normal_bf16_device((M, N), 0.01, 0, "llama65b", base + 4, device=dev)
        q0 = qb.NF4Weight.empty(N, K, dev)
        nq = max(2, math.ceil(2 * l2 / (0.515869 * N * K)))
        qs = [q0] + [qb.NF4Weight.empty(N, K, dev) for _ in range(nq - 1)]
        qcs = [q.as_c() for q in qs]
        Wd = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        T = torch.empty(M, R, dtype=torch.float32, device=dev)
        dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
        dA = torch.empty(R, K, dtype=torch.bfloat16, device=dev)
        dB = torch.empty(N, R, dtype=torch.bfloat16, device=dev)
        Y1 = torch.empty(1, N, dtype=torch.bfloat16, device=dev)
        X1 = X[:1].contiguous()
        need = 0
        for qc in qcs[:1]:
            n = ctypes.c_size_t(0)
            lib.qlora_quantize_nf4_dq(qb._ptr(W), ctypes.byref(qc), None, ctypes.byref(n), st)
            need = max(need, n.value)
            lib.qlora_linear_fwd(ctypes.byref(qc), qb._ptr(X), M, qb._ptr(A), qb._ptr(B), R, ALPHA, qb._ptr(Y),
                                 qb._ptr(T), None, ctypes.byref(n), st)
            need = max(need, n.value)
            lib.qlora_linear_bwd(ctypes.byref(qc), qb._ptr(X), M, qb._ptr(A), qb._ptr(B), R, ALPHA, qb._ptr(dY),
                                 qb._ptr(T), qb._ptr(dX), qb._ptr(dA), qb._ptr(dB), None, ctypes.byref(n), st)
            need = max(need, n.value)
            lib.qlora_linear_fwd(ctypes.byref(qc), qb._ptr(X1), 1, qb._ptr(A), qb._ptr(B), R, ALPHA, qb._ptr(Y1),
                                 None, None, ctypes.byref(n), st)
            need = max(need, n.value)
        wsb = torch.empty(need, dtype=torch.uint8, device=dev)
        ws, n = ctypes.c_void_p(wsb.data_ptr()), ctypes.c_size_t(need)
        for qc in qcs:  # every copy holds the quantized weight
            lib.qlora_quantize_nf4_dq(qb._ptr(W), ctypes.byref(qc), ws, ctypes.byref(n), st)
        us_q = _timed_calls([lambda qc=qc: lib.qlora_quantize_nf4_dq(qb._ptr(W), ctypes.byref(qc), ws,
                                                                      ctypes.byref(n), st) for qc in qcs], reps)
        us_d = _timed_calls([lambda qc=qc: lib.qlora_dequantize_nf4_dq(ctypes.byref(qc), qb._ptr(Wd), st)
                             for qc in qcs], reps)
        us_dec = _timed_calls([lambda qc=qc: lib.qlora_linear_fwd(
            ctypes.byref(qc), qb._ptr(X1), 1, qb._ptr(A), qb._ptr(B), R, ALPHA, qb._ptr(Y1), None, ws,
            ctypes.byref(n), st) for qc in qcs], 3 * reps)
        qc = qcs[0]
        us_f = _timed_calls([lambda: lib.qlora_linear_fwd(ctypes.byref(qc), qb._ptr(X), M, qb._ptr(A), qb._ptr(B),
                                                          R, ALPHA, qb._ptr(Y), qb._ptr(T), ws, ctypes.byref(n),
                                                          st)], reps)
        us_b = _timed_calls([lambda: lib.qlora_linear_bwd(ctypes.byref(qc), qb._ptr(X), M, qb._ptr(A), qb._ptr(B),
                                                          R, ALPHA, qb._ptr(dY), qb._ptr(T), qb._ptr(dX),
                                                          qb._ptr(dA), qb._ptr(dB), ws, ctypes.byref(n), st)], reps)
        ff, fb = train_flops(N, K, M)
        fl_tot += ff + fb
        us_tot += us_f + us_b
        key = f"{N}x{K}"
        gq = quant_bytes(N, K) / us_q / 1e3
        gd = quant_bytes(N, K) / us_d / 1e3
        gw = weight_bytes(N, K) / us_dec / 1e3
        out[f"quantize/{key}"] = {"us": round(us_q, 2), "GB_s": round(gq, 1), "hbm_frac": round(gq / peaks["hbm_gbs"], 4)}
        out[f"dequantize/{key}"] = {"us": round(us_d, 2), "GB_s": round(gd, 1),
                                    "hbm_frac": round(gd / peaks["hbm_gbs"], 4)}
        out[f"decode1/{key}"] = {"us": round(us_dec, 2), "weight_GB_s": round(gw, 1),
                                 "GB_s": round(decode_bytes(N, K, 1) / us_dec / 1e3, 1),
                                 "hbm_frac": round(decode_bytes(N, K, 1) / us_dec / 1e3 / peaks["hbm_gbs"], 4)}
        out[f"train_fwd/{key}"] = {"us": round(us_f, 2), "TFLOP_s": round(ff / us_f / 1e6, 1),
                                   "tensor_frac": round(ff / us_f / 1e6 / peaks["bf16_tflops"], 4)}
        out[f"train_bwd/{key}"] = {"us": round(us_b, 2), "TFLOP_s": round(fb / us_b / 1e6, 1),
                                   "tensor_frac": round(fb / us_b / 1e6 / peaks["bf16_tflops"], 4)}
        del W, A, B, X, dY, qs, qcs, Wd, Y, T, dX, dA, dB, wsb
        torch.cuda.empty_cache()
    err = qb.qlora_device_error()
    return {"workload": "Llama-65B linear shapes, W ~ Student-t(4) scaled to std 0.02, r=64 alpha=16, "
                        "train M=2048, decode M=1",
            "train_fwd_bwd_TFLOP_s": round(fl_tot / us_tot / 1e6, 1),
            "train_tensor_frac": round(fl_tot / us_tot / 1e6 / peaks["bf16_tflops"], 4),
            "parts": out, "device_error": err}


def measure_sweep65b(dev, peaks):
    """The 80-layer Llama-65B sweep (560 linears, 64.76e9 weights ~ N(0, 0.02)
    drawn on the device layer by layer): quantize + DQ of every linear into resident
    NF4 storage (33.4 GB), then one dequant pass and one M = 1 decode pass over all
    560 linears. Quantize time is the sum of per-layer event pairs around the seven
    calls of a layer (the weight generation stays outside them)."""
    import ctypes
    lib = qb.load_library()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    shapes = syn.LLAMA65B_LAYER
    nlin = len(shapes)
    layer_numel = sum(N * K for N, K in shapes)
    wbuf = torch.empty(layer_numel, dtype=torch.bfloat16, device=dev)
    offs, o = [], 0
    for N, K in shapes:
        offs.append(o)
        o += N * K
    need = 0
    for N, K in shapes:  # workspace size queries (nothing is launched)
        qq = qb.NF4Weight.empty(N, K, dev)
        qc = qq.as_c()
        n = ctypes.c_size_t(0)
        X1 = torch.empty(1, K, dtype=torch.bfloat16, device=dev)
        if lib.qlora_quantize_nf4_dq(qb._ptr(X1), ctypes.byref(qc), None, ctypes.byref(n), st) != 0:
            raise qb.QloraError(1, "sweep workspace query")
        need = max(need, n.value)
        if lib.qlora_linear_fwd(ctypes.byref(qc), qb._ptr(X1), 1, qb._ptr(X1), qb._ptr(X1), R, ALPHA, qb._ptr(X1),
                                None, None, ctypes.byref(n), st) != 0:
            raise qb.QloraError(1, "sweep workspace query")
        need = max(need, n.value)
        del qq, X1
    wsb = torch.empty(need, dtype=torch.uint8, device=dev)
    ws, n = ctypes.c_void_p(wsb.data_ptr()), ctypes.c_size_t(need)
    stor, qcs = [], []
    us_q = 0.0
    for layer in range(syn.LLAMA65B_LAYERS):
        for j, (N, K) in enumerate(shapes):
            syn.normal_bf16_device((N, K), 0.02, 0, "sweep65b", 16 * (nlin * layer + j), device=dev,
                                   out=wbuf[offs[j]:offs[j] + N * K].view(N, K))
        lq = [qb.NF4Weight.empty(N, K, dev) for N, K in shapes]
        lc = [q.as_c() for q in lq]
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for j in range(nlin):
            rc = lib.qlora_quantize_nf4_dq(qb._ptr(wbuf[offs[j]:]), ctypes.byref(lc[j]), ws, ctypes.byref(n), st)
            if rc != 0:
                raise qb.QloraError(rc, "sweep quantize")
        b.record()
        torch.cuda.synchronize()
        us_q += 1e3 * a.elapsed_time(b)
        stor.extend(lq)
        qcs.extend(lc)
    del wbuf
    torch.cuda.empty_cache()
    stored = sum(t.numel() * t.element_size() for q in stor for t in (q.packed, q.absmax_q, q.dq_scale, q.mean))
    nmax = max(N * K for N, K in shapes)
    dq_out = torch.empty(nmax, dtype=torch.bfloat16, device=dev)
    A_l = [syn.normal_bf16_device((R, K), 0.02, 0, "sweep65b", 9000 + 4 * j, device=dev) for j, (N, K) in
           enumerate(shapes)]
    B_l = [syn.normal_bf16_device((N, R), 0.02, 0, "sweep65b", 9001 + 4 * j, device=dev) for j, (N, K) in
           enumerate(shapes)]
    X_l = [syn.normal_bf16_device((1, K), 1.0, 0, "sweep65b", 9002 + 4 * j, device=dev) for j, (N, K) in
           enumerate(shapes)]
    Y_l = [torch.empty(1, N, dtype=torch.bfloat16, device=dev) for N, K in shapes]

    def dequant_all():
        for i, qc in enumerate(qcs):
            rc = lib.qlora_dequantize_nf4_dq(ctypes.byref(qc), qb._ptr(dq_out), st)
            if rc != 0:
                raise qb.QloraError(rc, "sweep dequant")

    def decode_all():
        for i, qc in enumerate(qcs):
            j = i % nlin
            rc = lib.qlora_linear_fwd(ctypes.byref(qc), qb._ptr(X_l[j]), 1, qb._ptr(A_l[j]), qb._ptr(B_l[j]), R,
                                      ALPHA, qb._ptr(Y_l[j]), None, ws, ctypes.byref(n), st)
            if rc != 0:
                raise qb.QloraError(rc, "sweep decode")

    res = {}
    for name, fn in (("dequant_all", dequant_all), ("decode1_all", decode_all)):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        res[name] = 1e3 * a.elapsed_time(b)
    err = qb.qlora_device_error()
    nw = syn.LLAMA65B_LAYERS * layer_numel
    lora_bytes = syn.LLAMA65B_LAYERS * sum(2 * R * (K + N) + 2 * (K + N) for N, K in shapes)
    gq = 2.516 * nw / us_q / 1e3
    gd = 2.516 * nw / res["dequant_all"] / 1e3
    gw = stored / res["decode1_all"] / 1e3
    gall = (stored + lora_bytes) / res["decode1_all"] / 1e3
    out = {"workload": "80 layers x 7 Llama-65B linears (560), 64.76e9 weights ~ N(0, 0.02) drawn on the device; "
                       "r=64 adapters per linear shape; decode M=1",
           "weights": nw, "nf4_bytes": stored,
           "quantize_all": {"ms": round(us_q / 1e3, 3), "GB_s": round(gq, 1), "hbm_frac": round(gq / peaks["hbm_gbs"], 4)},
           "dequant_all": {"ms": round(res["dequant_all"] / 1e3, 3), "GB_s": round(gd, 1),
                           "hbm_frac": round(gd / peaks["hbm_gbs"], 4)},
           "decode1_all": {"ms": round(res["decode1_all"] / 1e3, 3), "weight_GB_s": round(gw, 1),
                           "GB_s": round(gall, 1), "hbm_frac": round(gall / peaks["hbm_gbs"], 4)},
           "device_error": err}
    del stor, qcs, dq_out, A_l, B_l, X_l, Y_l, wsb
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, dev):
    def say(msg):  # progress on stderr (stdout carries only the JSON line)
        if args.verbose or rank == 0:
            print(f"[bench rank {rank}] {msg}", file=sys.stderr, flush=True)

    peaks = load_peaks()
    say("allocating the workload")
    dp = world > 1
    work = Workload(dev, seed=rank, dp=dp)
    fl_train = sum(sum(train_flops(N, K)) for N, K in SHAPES)

    clocks = ClockSampler(gpu_index_for_smi(dev))
    clocks.start()
    say("warm-up")
    t_w = time.time()
    for i in range(args.warmup):
        work.step()
        if i == 0:
            torch.cuda.synchronize()
            # a kernel wait that gave up (device error word) makes every later
            # number meaningless: stop here, on every rank, instead of timing it
            if max_over_ranks(float(qb.qlora_device_error()), world, dev):
                raise RuntimeError(f"device error {qb.qlora_device_error()} after the first warm-up step")
    while time.time() - t_w < 1.0:  # let the sampler produce its first lines
        work.step()
        torch.cuda.synchronize()
    torch.cuda.synchronize()

    # timed region: K whole steps; events on the launching stream bracket the region
    say("timed region (stream launches)")
    barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks.mark_begin()
    t0.record()
    for _ in range(args.steps):
        work.step()
    t1.record()
    torch.cuda.synchronize()
    barrier(world)
    ms_eager = max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)

    # the same step captured once into a CUDA graph (the library's launches keep
    # their programmatic-dependent-launch edges) and replayed K times
    ms_graph = None
    if not args.no_graph and not dp:  # the data-parallel step (NCCL on a side stream) runs as stream launches
        say("timed region (CUDA graph replay)")
        graph = capture_step_graph(work, say)
        # every rank takes the same collective steps: replay only if all captured
        if world > 1 and max_over_ranks(0.0 if graph is not None else 1.0, world, dev) > 0.0:
            graph = None
        if graph is not None:
            for _ in range(3):
                graph.replay()
            torch.cuda.synchronize()
            barrier(world)
            torch.cuda.synchronize()
            g0 = torch.cuda.Event(enable_timing=True)
            g1 = torch.cuda.Event(enable_timing=True)
            g0.record()
            for _ in range(args.steps):
                graph.replay()
            g1.record()
            torch.cuda.synchronize()
            barrier(world)
            ms_graph = max_over_ranks(g0.elapsed_time(g1) / args.steps, world, dev)
            del graph

    # the roofline call: K more whole steps, with an event pair around the
    # dominant call of each (and a device spin before it, so that the pair
    # brackets device execution only)
    say("roofline call inside K steps")
    li_roof = SHAPES.index(ROOFLINE_SHAPE)
    roof_part = f"train_fwd/{li_roof}"
    ev = {}
    for _ in range(args.steps):
        work.step(ev, only={roof_part})
    torch.cuda.synchronize()
    clocks.mark_end()
    clk = clocks.stop()
    ms_step = ms_graph if ms_graph is not None else ms_eager
    err = qb.qlora_device_error()

    # per-part breakdown (outside the timed region): each call run back to back,
    # cycling through enough copies of its inputs and outputs to exceed twice the
    # L2, so that every call reads its weights from HBM
    say("per-part breakdown")
    part_us = breakdown(work, dev)
    parts = {}
    for part, us in part_us.items():
        kind, li = part.split("/")
        N, K = SHAPES[int(li)]
        e = {"us": round(us, 2)}
        single = kind.endswith("_single")
        base = kind[: -len("_single")] if single else kind
        if base in ("quantize", "dequantize"):
            e["GB_s"] = round(quant_bytes(N, K, single) / us / 1e3, 1)
        elif base.startswith("decode"):
            M = int(base[len("decode"):])
            e["GB_s"] = round(decode_bytes(N, K, M, single=single) / us / 1e3, 1)
            e["weight_GB_s"] = round(weight_bytes(N, K, single) / us / 1e3, 1)
        else:
            f = train_flops(N, K)[0 if kind == "train_fwd" else 1]
            e["TFLOP_s"] = round(f / us / 1e6, 1)
        parts[f"{kind}/{N}x{K}"] = e

    # dominant call: the training forward (M = 4096) on the 11008x4096 linear, i.e.
    # one dequant, the LoRA-down GEMM + finish and the 2-CTA tcgen05 GEMM with the
    # LoRA slab; algorithmic flops over its measured duration (events on the stream).
    # median over the K calls: a call that met a power-capped clock dip does not move it
    fwd_us = 1e3 * statistics.median(a.elapsed_time(b) for a, b in ev[roof_part])
    achieved = train_flops(*ROOFLINE_SHAPE)[0] / fwd_us / 1e6
    traffic = TRAFFIC_RECORD["bytes"] if TRAFFIC_RECORD["fingerprint"] == source_fingerprint() else None
    # the call is timed alone (its own event pair, a few hundred microseconds), so
    # the burst figure is its peak; the sustained one is reported beside it
    roof = {"kernel": "qlora_linear_fwd M=4096 on 11008x4096 (dequant, LoRA-down, 2-CTA tcgen05 GEMM)",
            "bound": "tensor", "achieved": round(achieved, 1), "peak": peaks["bf16_tflops"],
            "peak_kind": f"bf16 dense burst ({peaks['source']})", "unit": "TFLOP/s",
            "frac": round(achieved / peaks["bf16_tflops"], 4),
            "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4), "traffic": traffic,
            "us_per_launch": round(fwd_us, 2)}
    dec = [parts[f"decode{M}/{N}x{K}"]["weight_GB_s"] for M in M_DECODE for N, K in SHAPES]

    say("adapter merge")
    merge = merge_measure(work, dev)
    say("paged AdamW")
    adamw = adamw_measure(dev, peaks)
    llama65b = sweep = None
    if not args.no_65b:
        say("Llama-65B shapes (Student-t weights)")
        llama65b = measure_llama65b(dev, peaks)
        say("80-layer Llama-65B sweep")
        sweep = measure_sweep65b(dev, peaks)
    say("end to end with host buffers")
    # end to end through the C ABI with host buffers
    host = []
    for d in work.lin:
        h = {k: torch.empty_like(d[k], device="cpu").pin_memory() for k in ("W", "A", "B", "X", "dY")}
        for k in h:
            h[k].copy_(d[k])
        for k in (("grads_bf16",) if work.dp else ("dA", "dB")):
            h["out_" + k] = torch.empty_like(d[k], device="cpu").pin_memory()
        for M in M_DECODE:
            h[f"out_Y{M}"] = torch.empty_like(d["Ydec"][M], device="cpu").pin_memory()
        host.append(h)
    e2e_steps = max(1, min(args.steps, 5))
    streams = E2EStreams(len(work.lin))
    e2e_step(work, host, streams)
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(e2e_steps):
        h2d, d2h = e2e_step(work, host, streams, start=e0 if i == 0 else None)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)

    value = world * fl_train / (ms_step * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "launch": "CUDA graph replay of the step" if ms_graph is not None else "stream launches",
        "ms_per_step_stream_launches": round(ms_eager, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, per-rank seed)",
        "config": {"workload": "Llama-7B linear shapes 4096x4096, 11008x4096, 4096x11008; r=64 alpha=16; "
                               "quantize+DQ, dequant, decode M=1/4/16, train fwd+bwd M=4096",
                   "global_batch_tokens": M_TRAIN * world,
                   "parallelism": (f"dp{world} (token shards of {M_TRAIN} per rank; fp32 LoRA gradients all-reduced "
                                   "over NCCL on a side stream, overlapping the dX GEMM)") if dp else "dp1 (one GPU)",
                   "l2": "inputs larger than L2 (each step touches ~1.2 GB)",
                   "parts": "each call back to back over rotating input copies > 2x L2, outside the timed region"},
        "decode_weight_GB_s": {"min": min(dec), "max": max(dec)},
        "hbm_frac": {k: round(v["GB_s"] / peaks["hbm_gbs"], 4) for k, v in parts.items() if "GB_s" in v},
        "parts": parts,
        "roofline": roof,
        "merge": merge,
        "adamw": adamw,
        "llama65b": llama65b,
        "sweep65b": sweep,
        "e2e": {"value": round(world * fl_train / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": work.launches_per_step() * args.steps,
        "clocks": clk,
        "device_error": err,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_sample(seconds_budget=args.cpu_seconds)
    return line


# ----------------------------------------------------------------------------
# oracle (CPU) arm

def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 1) for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def oracle_step_sample(N=4096, K=4096, M=256, seed=0):
    """One pass of the hot path on one linear, computed by the CPU oracle:
    quantize + DQ, dequant, decode M = 1/4/16 and forward + backward at M tokens."""
    import numpy as np
    import oracle
    inp = syn.make_linear(N, K, M, r=R, alpha=ALPHA, seed=seed, workload="llama7b_train", layer=0)
    f64 = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
    Wf = inp.W.float().numpy()
    X, A, B, dY = f64(inp.X), f64(inp.A), f64(inp.B), f64(inp.dY)
    t = time.perf_counter()
    qw = oracle.quantize_nf4_dq(Wf)
    Wd = oracle.bf16_bits_to_f32(oracle.dequantize_nf4_dq(qw)).astype(np.float64)
    s = oracle.lora_scale(ALPHA, R)
    for Md in M_DECODE:
        oracle.linear_fwd(Wd, X[:Md], A, B, s)
    oracle.linear_fwd(Wd, X, A, B, s)
    oracle.linear_bwd(Wd, X, A, B, dY, s)
    dt = time.perf_counter() - t
    return sum(train_flops(N, K, M)), dt


def cpu_baseline_sample(seconds_budget=20.0):
    fl, dt = oracle_step_sample()
    reps = 1
    while dt * (reps + 1) / reps < seconds_budget and reps < 8 and dt < seconds_budget / 2:
        f2, d2 = oracle_step_sample(seed=reps)
        fl += f2
        dt += d2
        reps += 1
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
            "sample": f"{reps} x one pass of the hot path on the 4096x4096 linear (quantize+DQ, dequant, "
                      f"decode M=1/4/16, fwd+bwd at M=256 in fp64); value = fwd+bwd flops / total oracle time",
            "seconds": round(dt, 2)}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    for _ in range(args.warmup):
        oracle_step_sample(M=64)
    fl = 0.0
    t0 = time.perf_counter()
    for i in range(args.steps):
        f, _ = oracle_step_sample(seed=i)
        fl += f
    dt = time.perf_counter() - t0
    v = fl / dt / 1e12
    return {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * dt / args.steps, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "one pass of the hot path on the 4096x4096 Llama-7B linear per step "
                                   "(bounded sample of the GPU arm's workload), train M=256, r=64 alpha=16"},
            "cpu_baseline": {"value": round(v, 6), "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
                             "sample": "per step: quantize+DQ, dequant, decode M=1/4/16, fwd+bwd M=256 on 4096x4096"},
            "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------
# small profiling case (for ncu captures): one call of each entry point on the
# 11008x4096 linear, training M = 4096 and decode M = 1

def profile_case():
    dev = torch.device("cuda", 0)
    N, K = 11008, 4096
    inp = syn.make_linear(N, K, M_TRAIN, r=R, alpha=ALPHA, seed=0, workload="llama7b_train", layer=1)
    W, A, B, X, dY = (t.to(dev) for t in (inp.W, inp.A, inp.B, inp.X, inp.dY))
    q = qb.qlora_quantize_nf4_dq(W)                                   # quantize + DQ
    qb.qlora_dequantize_nf4_dq(q)                                     # dequant
    qb.qlora_linear_fwd(q, X[:1].contiguous(), A, B, ALPHA)           # decode M = 1
    qb.qlora_linear_fwd(q, X[:16].contiguous(), A, B, ALPHA)          # decode M = 16
    _, T = qb.qlora_linear_fwd(q, X, A, B, ALPHA, T_save=True)        # training forward
    qb.qlora_linear_bwd(q, X, A, B, ALPHA, dY, T_saved=T)             # training backward
    torch.cuda.synchronize()
    assert qb.qlora_device_error() == 0
    print("profile case ok")


# ----------------------------------------------------------------------------
# distributed plumbing

def gpu_index_for_smi(dev):
    """Physical index of `dev` for nvidia-smi (honours CUDA_VISIBLE_DEVICES)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if dev.index < len(ids) and ids[dev.index].isdigit():
            return int(ids[dev.index])
    return dev.index

def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, dev):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print progress to stderr")
    ap.add_argument("--no-graph", action="store_true", help="time stream launches only (no CUDA graph replay)")
    ap.add_argument("--no-65b", action="store_true", help="skip the Llama-65B shape and 80-layer sweep measurements")
    ap.add_argument("--profile-case", action="store_true",
                    help="run one call of each entry point on 11008x4096 (for ncu) and exit")
    args = ap.parse_args()
    if args.profile_case:
        qb.load_library()
        profile_case()
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: WORLD_SIZE={world} but --gpus={args.gpus}", file=sys.stderr)
    if args.impl == "reference":
        if world > 1:
            torch.distributed.init_process_group("gloo", timeout=__import__("datetime").timedelta(seconds=600))
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=dev)
    qb.load_library()
    line = run_ours(args, rank, world, dev)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
