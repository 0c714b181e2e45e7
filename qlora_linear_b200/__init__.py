"""LoRA-adapted linear layer over a frozen bf16 or 4-bit blockwise weight, for B200.

The compute lives in ``liblora_linear.so`` (hand-written sm_100a CUDA behind a C ABI,
``include/lora_linear.h``); this package is its ctypes binding plus a small layer
object that allocates outputs with torch.  Importing fails loudly when the library
has not been built.
"""
from .binding import (  # noqa: F401
    EXPORTED,
    LIB_PATH,
    LORA_ERR_ALIGNMENT,
    LORA_ERR_CUDA,
    LORA_ERR_DEVICE_TIMEOUT,
    LORA_ERR_INVALID_ARG,
    LORA_ERR_UNSUPPORTED,
    LORA_ERR_WORKSPACE,
    LORA_OK,
    LORA_W_BF16,
    LORA_W_BLOCK4,
    LORA_W_INT8,
    LORA_W_FP8_E4M3,
    lora_dequant,
    LoraError,
    LoraWeight,
    alloc_workspace,
    dequant_blockwise4,
    lib,
    lora_device_status,
    lora_linear_bwd,
    lora_linear_fwd,
    lora_linear_fwd_noalloc,
    lora_grouped_fwd,
    lora_grouped_bwd,
    grouped_workspace_bytes,
    lora_mlp_fwd,
    lora_mlp_bwd,
    lora_mlp_t,
    mlp_struct,
    mlp_workspace_bytes,
    segments,
    LORA_ERR_SCRATCH_LIMIT,
    LORA_NOALLOC_SCRATCH_BYTES,
    lora_merge,
    lora_testing_bounded_wait,
    LORA_KERNEL_BWD_GEMM,
    LORA_KERNEL_FWD_GEMM,
    lora_launch_count,
    lora_timing_enable,
    lora_timing_read,
    status_string,
    workspace_bytes,
)
from .layer import LoraGroupedLinear, LoraLinear, LoraMLP  # noqa: F401
from .dp import allreduce_adapter_grads, token_shard  # noqa: F401
