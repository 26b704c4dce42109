"""B200 (sm_100a) QLoRA NF4 library: NF4 block-wise absmax quantization,
double quantization of the absmax constants, dequantization and the QLoRA
linear layer forward/backward, behind the C ABI of include/qlora.h.

The compute runs in ``libqlora_b200.so`` (hand-written CUDA); ``binding``
marshals torch tensors into it. Importing this package does not load the
library; the first call does, and fails loudly if it has not been built.
"""
from .binding import (NF4Weight, QloraError, load_library, qlora_device_error, qlora_dequantize_nf4_dq,
                      qlora_linear_bwd, qlora_linear_fwd, qlora_nf4_codebook, qlora_nf4_storage_bytes,
                      qlora_quantize_nf4_dq, qlora_status_string)

__all__ = ["NF4Weight", "QloraError", "load_library", "qlora_device_error", "qlora_dequantize_nf4_dq",
           "qlora_linear_bwd", "qlora_linear_fwd", "qlora_nf4_codebook", "qlora_nf4_storage_bytes",
           "qlora_quantize_nf4_dq", "qlora_status_string"]
