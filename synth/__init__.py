"""Seeded synthetic inputs for the LoRA-adapted linear layer.

This package is shared by the tests, ``bench.py`` and ``__graft_entry__.smoke()``.
It holds random draws and their rounding to the storage types only; none of the
layer's arithmetic lives here.
"""
from .inputs import (  # noqa: F401
    CONFIGS,
    LoraCase,
    bf16_bits_from_f32,
    f32_from_bf16_bits,
    make_case,
    make_grouped_case,
    MlpCase,
    make_mlp_case,
    CeCase,
    make_ce_case,
    config_cases,
)
