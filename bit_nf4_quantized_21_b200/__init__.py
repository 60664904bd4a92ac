"""QLoRA frozen-base NF4 linear layer for NVIDIA B200 (sm_100a).

The compute lives in libqlora.so (hand-written CUDA behind a C ABI,
include/qlora.h); ``bit_nf4_quantized_21_b200.qlora`` is its ctypes binding
and ``bit_nf4_quantized_21_b200.inputs`` draws the seeded synthetic inputs.
The library is loaded on first use; calls raise if it has not been built.
"""
from .qlora import (  # noqa: F401
    NF4Weight, QloraError, empty_nf4, lib, qlora_dequantize, qlora_linear_bwd, qlora_linear_fwd,
    qlora_adam_step, qlora_merge_nf4, qlora_linear_fwd_noalloc, qlora_lora_linear_bwd, qlora_lora_linear_fwd, qlora_nf4_codebook,
    qlora_nf4_sizes, qlora_quantize_nf4, qlora_workspace_bytes, status_string,
    qlora_workspace_bytes_dropout, qlora_lora_dropout_mask, qlora_linear_fwd_dropout, qlora_linear_bwd_dropout,
    qlora_paged_alloc, qlora_paged_free, qlora_paged_prefetch,
)

__version__ = "0.1.0"
