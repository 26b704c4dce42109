"""CPU oracle for the QLoRA NF4 + double-quant + LoRA linear hot path.

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the test suite, the smoke check of
``__graft_entry__`` and the CPU-baseline / reference legs of ``bench.py`` may
import or run anything in this package. The library's CUDA path shares no code
with it, and it imports nothing from the library.

The oracle is deliberately plain and slow: numpy/Python on the host, fp64 for
every real-valued reduction and GEMM, and exact (integer or rational) arithmetic
wherever a rounding decides a stored bit pattern. Each function cites the web
page passage it follows:

* "Guanaco" (chipfoundryservices.com/topic/guanaco), sections "Core
  Architecture & Training" and "Technical Innovations".
* "QLoRA: Efficient Finetuning of Quantized LLMs" (ai-papercheck.pages.dev
  errata list), findings quoting the paper's p.4 Section 2 and p.5 Section 3.
* "QLoRA vs ChatGPT" (unfragile.ai compare page), capability blurbs 1 (NF4 with
  block-wise absmax), 2 (LoRA on a frozen 4-bit base), 3 (double quantization,
  contrasted with single-level constants; the errata page's p.8 Table 4
  findings compare NFloat4 with and without DQ),
  4 (paged optimizers), 5 (training pipeline: block-wise on-the-fly
  dequantization, gradients for the LoRA parameters only) and 6 (composing
  adapters and merging them into the base weights).

Where the pages are silent the oracle takes one stated reading; every reading is
listed in the repository's design notes.
"""
from .fp import bf16_bits_to_f32, f32_to_bf16_bits_rn, fma_f32
from .nf4 import (BLOCK, DQ_BLOCK, nf4_codebook, fp4_codebook, quantize_nf4, dq_mean, double_quantize, quantize_nf4_dq,
                  dequantize_nf4_dq, pack_codes, unpack_codes, storage_bytes, QuantizedNF4, QuantizedNF4Single,
                  quantize_nf4_single, dequantize_nf4_single)
from .linear import lora_scale, linear_fwd, linear_bwd, linear_fwd_multi
from .merge import f64_to_bf16_bits_rn, merge_lora, merge_scale
from .optim import adamw_step

__all__ = [
    "bf16_bits_to_f32", "f32_to_bf16_bits_rn", "fma_f32",
    "BLOCK", "DQ_BLOCK", "nf4_codebook", "fp4_codebook", "quantize_nf4", "dq_mean", "double_quantize", "quantize_nf4_dq",
    "dequantize_nf4_dq", "pack_codes", "unpack_codes", "storage_bytes", "QuantizedNF4", "QuantizedNF4Single",
    "quantize_nf4_single", "dequantize_nf4_single",
    "lora_scale", "linear_fwd", "linear_bwd", "linear_fwd_multi",
    "f64_to_bf16_bits_rn", "merge_lora", "merge_scale", "adamw_step",
]
