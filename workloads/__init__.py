"""Seeded synthetic workloads for causal scaled-dot-product attention.

This package only draws inputs: random tensors, packed-document boundaries and
the caller-side RoPE sin/cos tables. It holds none of the attention arithmetic,
so both the CPU oracle and the CUDA path can take their inputs from it without
sharing any of the method's code.
"""

from .configs import CONFIGS, Config, config_by_name
from .decode import (
    DECODE_CONFIGS,
    DecodeConfig,
    DecodeWorkload,
    decode_config_by_name,
    make_decode_workload,
)
from .projection import (
    PROJ_CONFIGS,
    ProjConfig,
    ProjWorkload,
    make_proj_workload,
    proj_config_by_name,
)
from .generate import (
    Workload,
    draw_doc_lengths,
    make_workload,
    rope_tables_f32,
    round_to_bf16,
)

__all__ = [
    "CONFIGS",
    "DECODE_CONFIGS",
    "DecodeConfig",
    "DecodeWorkload",
    "decode_config_by_name",
    "make_decode_workload",
    "PROJ_CONFIGS",
    "ProjConfig",
    "ProjWorkload",
    "make_proj_workload",
    "proj_config_by_name",
    "Config",
    "Workload",
    "config_by_name",
    "draw_doc_lengths",
    "make_workload",
    "rope_tables_f32",
    "round_to_bf16",
]
