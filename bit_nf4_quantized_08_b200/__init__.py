"""QLoRA NF4 frozen linear layer for NVIDIA B200 (sm_100a).

``Y = X dequant_NF4(W_q)^T + (alpha/r) (X A^T) B^T``, its backward (dX, dA,
dB; never dW), and the blockwise NF4 quantizer with 8-bit double
quantization of the block constants, as a C-ABI CUDA library
(``include/qlora_nf4.h``) with a thin torch binding.
"""
from ._lib import QloraError, QLORA_OK, QLORA_ERR_INVALID_ARG, QLORA_ERR_UNSUPPORTED, \
    QLORA_ERR_CUDA, QLORA_ERR_TIMEOUT, QLORA_ERR_WORKSPACE, QLORA_ERR_BOUNDS, QLORA_STATIC_QUANTIZE_MAX_ELEMS  # noqa: F401
from .api import (  # noqa: F401
    NF4Weight,
    PagedBuffer,
    qlora_adamw_step,
    qlora_debug_inject,
    qlora_dq_encode,
    qlora_fused_linear_bwd,
    qlora_fused_linear_fwd,
    qlora_fused_linear_workspace,
    qlora_get_last_error,
    qlora_linear_bwd,
    qlora_linear_fwd,
    qlora_linear_workspace,
    qlora_lora_merge,
    qlora_lora_unmerge,
    qlora_nf4_dequantize,
    qlora_nf4_encode,
    qlora_nf4_quantize,
    qlora_nf4_quantize_static,
    qlora_nf4_quantize_workspace,
    qlora_nf4_table,
    qlora_set_wait_timeout_ns,
    qlora_kernel_launches,
    qlora_profile_enable,
    qlora_profile_read,
)
