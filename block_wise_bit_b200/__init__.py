"""block_wise_bit_b200 -- block-wise 8-bit optimizer state on NVIDIA B200 (sm_100a).

The C ABI (include/bnbq.h, libbnbq.so) holds the hot path: block-wise dynamic quantize /
dequantize (8-bit and NF4) and the fused multi-tensor 8-bit AdamW / Adam / Lion / momentum /
RMSprop step.  ``bindings`` is its ctypes marshalling layer (same names as the C entry points);
``optim`` holds the launcher policy (which tensors keep 32-bit state) and torch.optim-style
front ends; ``workloads`` describes seeded synthetic parameter lists.
"""
from .bindings import (BnbqError, TensorState, bnbq_check_codebook, bnbq_codebook, bnbq_dequantize_absmax_nested,
                       bnbq_dequantize_blockwise, bnbq_dequantize_blockwise_nested, bnbq_device_flags,
                       bnbq_last_error, bnbq_quantize_absmax_nested, bnbq_quantize_blockwise, bnbq_release,
                       bnbq_step_8bit, bnbq_version, lib, pack_tensor_list)

__all__ = ["BnbqError", "TensorState", "bnbq_check_codebook", "bnbq_codebook", "bnbq_dequantize_absmax_nested",
           "bnbq_dequantize_blockwise", "bnbq_dequantize_blockwise_nested", "bnbq_device_flags", "bnbq_last_error",
           "bnbq_quantize_absmax_nested", "bnbq_quantize_blockwise", "bnbq_release", "bnbq_step_8bit",
           "bnbq_version", "lib", "pack_tensor_list"]
