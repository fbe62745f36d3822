"""The five attention workloads, named by what they are.

Shapes and distributions follow the training-layer shapes the source pages
describe (a 12M GPT at context 512 in the Forge README, the 237M EKO decoder at
seq 1024 in the ARK README, 2K-8K training windows and packed short documents in
the Cort33x notes); the head counts, seeds and value scales are fixed here, per
workload, so that every run of the tests and the bench draws the same inputs.
"""

from __future__ import annotations

import math
from dataclasses import dataclass


@dataclass(frozen=True)
class Config:
    name: str
    dtype: str          # "f32" or "bf16": storage and I/O type of q, k, v, o, dO, dq, dk, dv
    B: int
    H: int
    T: int
    D: int
    rope: bool          # apply RoPE (theta below) to q and k
    theta: float
    varlen: bool        # pack documents of length Uniform[doc_min, doc_max] per row
    doc_min: int
    doc_max: int
    qk_std: float       # standard deviation of the q and k draws
    v_std: float
    do_std: float       # standard deviation of dO (0.01 reads "N(0, 0.01)" as a std)
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def nominal_flops(self) -> float:
        """fwd 4*B*H*T^2*D halved for causal, bwd 2.5x that: 7*B*H*T^2*D in total."""
        return 7.0 * self.B * self.H * self.T * self.T * self.D


CONFIGS = [
    Config("tiny_fp32", "f32", 1, 2, 128, 64, False, 10000.0, False, 0, 0,
           1.0, 1.0, 1.0, 0),
    Config("gpt12m_layer", "bf16", 16, 6, 512, 64, True, 10000.0, False, 0, 0,
           1.0, 1.0, 0.01, 1),
    Config("decoder237m_layer", "bf16", 8, 16, 1024, 64, True, 10000.0, False, 0, 0,
           1.5, 1.0, 0.01, 2),
    Config("long_context_8k", "bf16", 1, 16, 8192, 128, True, 10000.0, False, 0, 0,
           1.0, 1.0, 0.01, 3),
    Config("packed_docs", "bf16", 4, 16, 2048, 128, True, 10000.0, True, 32, 1024,
           1.0, 1.0, 0.01, 4),
]


def config_by_name(name: str) -> Config:
    for c in CONFIGS:
        if c.name == name:
            return c
    raise KeyError(f"unknown workload {name!r}; known: {[c.name for c in CONFIGS]}")
