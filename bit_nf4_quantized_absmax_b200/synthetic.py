"""Seeded synthetic inputs for the QLoRA NF4 linear workloads.

This module only draws random numbers; it holds none of the method's arithmetic
(no codebook, no quantization, no GEMM). Both the CUDA path and the CPU oracle
receive the tensors produced here as plain data.

Workloads (all tensors bf16, drawn in fp32 by torch's CPU generator and rounded
to bf16 to nearest-even by torch's own conversion):

* ``single``  : W 1024x1024 ~ N(0, 0.02); X 16x1024 ~ N(0, 1); r=16, alpha=16;
                A, B ~ N(0, 0.02); dY ~ N(0, 1).
* ``llama7b`` : W of the three Llama-7B linear shapes (out x in) 4096x4096,
                11008x4096, 4096x11008 ~ N(0, 0.02); r=64, alpha=16;
                A, B ~ N(0, 0.02); X ~ N(0, 1); dY ~ N(0, 0.01).
* ``llama65b``: W of the Llama-65B shapes 8192x8192, 22016x8192, 8192x22016
                drawn from Student-t(nu=4) scaled by 0.02/sqrt(2) (std 0.02,
                heavy tails); r=64, alpha=16; X ~ N(0, 1); dY ~ N(0, 0.01).

The second argument of every N(., .) above is a standard deviation.
Each tensor gets its own generator seeded from (seed, workload id, tensor id),
so any tensor can be regenerated alone.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

LLAMA7B_SHAPES = ((4096, 4096), (11008, 4096), (4096, 11008))
LLAMA65B_SHAPES = ((8192, 8192), (22016, 8192), (8192, 22016))

_WORKLOAD_IDS = {"single": 1, "llama7b": 2, "llama7b_train": 3, "llama65b": 4, "sweep65b": 5, "test": 9}


def tensor_seed(seed: int, workload: str, tensor_id: int) -> int:
    """Derive a 63-bit generator seed from (seed, workload, tensor id)."""
    wid = _WORKLOAD_IDS[workload]
    x = (seed * 0x9E3779B97F4A7C15 + wid * 0xBF58476D1CE4E5B9 + tensor_id * 0x94D049BB133111EB)
    return x & ((1 << 63) - 1)


def _gen(seed: int, workload: str, tensor_id: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(tensor_seed(seed, workload, tensor_id))
    return g


def normal_bf16(shape, std: float, seed: int, workload: str, tensor_id: int) -> torch.Tensor:
    """N(0, std) drawn in fp32 and rounded to bf16 (CPU tensor)."""
    g = _gen(seed, workload, tensor_id)
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def student_t_bf16(shape, nu: int, std: float, seed: int, workload: str, tensor_id: int) -> torch.Tensor:
    """Student-t(nu) samples scaled to the given std, rounded to bf16.

    Drawn from the textbook definition T = Z / sqrt(V / nu) with Z ~ N(0, 1)
    and V a chi-square with nu degrees of freedom (a sum of nu squared
    standard normals, nu integer). The t(nu) variance is nu / (nu - 2).
    """
    assert nu > 2 and int(nu) == nu
    g = _gen(seed, workload, tensor_id)
    z = torch.randn(*shape, generator=g, dtype=torch.float32)
    v = torch.zeros(*shape, dtype=torch.float32)
    for _ in range(int(nu)):
        e = torch.randn(*shape, generator=g, dtype=torch.float32)
        v.addcmul_(e, e)
    t = z / torch.sqrt(v / nu)
    t.mul_(std / math.sqrt(nu / (nu - 2.0)))
    return t.to(torch.bfloat16)


@dataclass
class LinearInputs:
    """One QLoRA linear problem: frozen W [N,K], adapters A [r,K], B [N,r],
    activations X [M,K] and upstream gradient dY [M,N] (all bf16, CPU)."""
    W: torch.Tensor
    A: torch.Tensor
    B: torch.Tensor
    X: torch.Tensor
    dY: torch.Tensor
    r: int
    alpha: float


def make_linear(N: int, K: int, M: int, r: int = 64, alpha: float = 16.0, *, seed: int = 0,
                workload: str = "llama7b", layer: int = 0, w_dist: str = "normal",
                x_std: float = 1.0, dy_std: float = 0.01, w_std: float = 0.02,
                lora_std: float = 0.02) -> LinearInputs:
    """Generate one linear's inputs. ``layer`` selects a distinct stream per linear."""
    base = 16 * layer
    if w_dist == "normal":
        W = normal_bf16((N, K), w_std, seed, workload, base + 0)
    elif w_dist == "student_t4":
        W = student_t_bf16((N, K), 4, w_std, seed, workload, base + 0)
    else:
        raise ValueError(w_dist)
    A = normal_bf16((r, K), lora_std, seed, workload, base + 1)
    B = normal_bf16((N, r), lora_std, seed, workload, base + 2)
    X = normal_bf16((M, K), x_std, seed, workload, base + 3) if M > 0 else torch.empty(0, K, dtype=torch.bfloat16)
    dY = normal_bf16((M, N), dy_std, seed, workload, base + 4) if M > 0 else torch.empty(0, N, dtype=torch.bfloat16)
    return LinearInputs(W, A, B, X, dY, r, alpha)


def _gen_cuda(seed: int, workload: str, tensor_id: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(tensor_seed(seed, workload, tensor_id))
    return g


def normal_bf16_device(shape, std: float, seed: int, workload: str, tensor_id: int, device="cuda",
                       out: torch.Tensor | None = None) -> torch.Tensor:
    """N(0, std) drawn on the device by torch's seeded (Philox) CUDA generator,
    rounded to bf16. Used where the workload is too large to draw on the host
    (the whole-model sweep); the values are reproducible for a given seed."""
    g = _gen_cuda(seed, workload, tensor_id, device)
    t = torch.randn(*shape, generator=g, dtype=torch.float32, device=device)
    t.mul_(std)
    if out is None:
        return t.to(torch.bfloat16)
    out.copy_(t)
    return out


def student_t_bf16_device(shape, nu: int, std: float, seed: int, workload: str, tensor_id: int,
                          device="cuda") -> torch.Tensor:
    """Student-t(nu) on the device (same definition as student_t_bf16), bf16."""
    assert nu > 2 and int(nu) == nu
    g = _gen_cuda(seed, workload, tensor_id, device)
    z = torch.randn(*shape, generator=g, dtype=torch.float32, device=device)
    v = torch.zeros(*shape, dtype=torch.float32, device=device)
    for _ in range(int(nu)):
        e = torch.randn(*shape, generator=g, dtype=torch.float32, device=device)
        v.addcmul_(e, e)
    t = z / torch.sqrt(v / nu)
    t.mul_(std / math.sqrt(nu / (nu - 2.0)))
    return t.to(torch.bfloat16)


# Per-layer linear shapes (out x in) of Llama-65B: q, k, v, o, gate, up, down.
LLAMA65B_LAYER = ((8192, 8192), (8192, 8192), (8192, 8192), (8192, 8192), (22016, 8192), (22016, 8192),
                  (8192, 22016))
LLAMA65B_LAYERS = 80


def single_linear(seed: int = 0) -> LinearInputs:
    """The 1024x1024 single-linear workload (r=16, alpha=16, dY ~ N(0,1))."""
    return make_linear(1024, 1024, 16, r=16, alpha=16.0, seed=seed, workload="single", dy_std=1.0)
