"""fp64 CPU oracle for the LoRA-adapted linear layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg use
this package.  It shares no code with the CUDA library and imports nothing from it.
"""
from .lora_oracle import (  # noqa: F401
    bf16_round_bits,
    bf16_to_f64,
    fp16_to_f64,
    lora_forward,
    lora_backward,
    lora_forward_rows,
    lora_backward_rows,
    dequant_blockwise4,
    quantize_blockwise4,
    nearest_codes,
    lora_merge,
    weight_f64,
    lora_adapter_grads_sampled,
    lora_grouped_forward,
    lora_grouped_backward,
    sigmoid,
    swiglu_forward,
    swiglu_backward,
    lora_mlp_forward,
    lora_mlp_backward,
    int8_value,
    e4m3_value,
    dequant_rowwise8,
    e4m3_nearest,
    quantize_rowwise8,
    cross_entropy,
    cross_entropy_rows_bits,
)
