"""Seeded workloads for the projections around the attention (no projection
or attention arithmetic lives here: only random draws).

Draw order from ``numpy.random.default_rng(seed)``, float32 standard normals
scaled by their standard deviations: x [B, T, C]; W_qkv [(H + 2 H_kv) D, C]
with std 1/sqrt(C) (the usual fan-in scale of a freshly initialised linear
layer); W_o [C, H D] with std 1/sqrt(H D); then the output gradients dq
[B, H, T, D], dk and dv [B, H_kv, T, D], d_y [B, T, C], each with std 0.01
(the attention workloads' dO convention); then, for packed rows, document
lengths Uniform[doc_lo, doc_hi] per row (last one truncated). Every tensor is
rounded to bf16 (RNE). The attention output o that the output projection
reads is drawn as standard normals too (its rows are convex combinations of
values, of the same scale).
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from .generate import draw_doc_lengths, rope_tables_f32, round_to_bf16


@dataclass(frozen=True)
class ProjConfig:
    name: str
    B: int
    T: int
    C: int      # model width
    H: int
    H_kv: int
    D: int
    rope: bool
    packed: bool
    seed: int
    doc_lo: int = 32
    doc_hi: int = 1024


PROJ_CONFIGS = [
    # the 237M decoder layer of the ARK README's parameter table: d_model 768,
    # 12 heads of 64, context 1024, batch of 8 sequences
    ProjConfig("proj_237m", 8, 1024, 768, 12, 12, 64, True, False, 30),
    # a long-context grouped-query layer: width 2048, 16 query heads of 128 on
    # 4 key/value heads, one 8K sequence
    ProjConfig("proj_gqa_8k", 1, 8192, 2048, 16, 4, 128, True, False, 31),
    # small parity cases with ragged widths (K and N tails) and packed documents
    ProjConfig("proj_small_d64", 2, 256, 200, 3, 1, 64, True, True, 32, 16, 100),
    ProjConfig("proj_small_d128", 2, 384, 136, 2, 1, 128, True, True, 33, 16, 100),
]


def proj_config_by_name(name: str) -> ProjConfig:
    for c in PROJ_CONFIGS:
        if c.name == name:
            return c
    raise KeyError(f"unknown projection workload {name!r}; known: {[c.name for c in PROJ_CONFIGS]}")


@dataclass
class ProjWorkload:
    cfg: ProjConfig
    x: np.ndarray
    w_qkv: np.ndarray
    w_o: np.ndarray
    o: np.ndarray
    dq: np.ndarray
    dk: np.ndarray
    dv: np.ndarray
    dy: np.ndarray
    rope_cos: Optional[np.ndarray]
    rope_sin: Optional[np.ndarray]
    cu_seqlens: Optional[np.ndarray]

    def flops(self) -> dict:
        """Multiply-add flops (2 per product term) of each GEMM."""
        c = self.cfg
        bt = c.B * c.T
        f = (c.H + 2 * c.H_kv) * c.D
        hd = c.H * c.D
        return {"qkv": 2.0 * bt * c.C * f, "qkv_bwd": 4.0 * bt * c.C * f,
                "out": 2.0 * bt * hd * c.C, "out_bwd": 4.0 * bt * hd * c.C}


def make_proj_workload(cfg: ProjConfig, *, B: Optional[int] = None, T: Optional[int] = None,
                       C: Optional[int] = None, H: Optional[int] = None,
                       H_kv: Optional[int] = None, D: Optional[int] = None,
                       rope: Optional[bool] = None, packed: Optional[bool] = None,
                       seed: Optional[int] = None) -> ProjWorkload:
    B = cfg.B if B is None else B
    T = cfg.T if T is None else T
    C = cfg.C if C is None else C
    H = cfg.H if H is None else H
    H_kv = cfg.H_kv if H_kv is None else H_kv
    D = cfg.D if D is None else D
    rope = cfg.rope if rope is None else rope
    packed = cfg.packed if packed is None else packed
    seed = cfg.seed if seed is None else seed
    cfg = ProjConfig(cfg.name, B, T, C, H, H_kv, D, rope, packed, seed, cfg.doc_lo, cfg.doc_hi)
    rng = np.random.default_rng(seed)
    f32 = np.float32
    x = rng.standard_normal((B, T, C), dtype=f32)
    w_qkv = rng.standard_normal(((H + 2 * H_kv) * D, C), dtype=f32) * f32(1.0 / np.sqrt(C))
    w_o = rng.standard_normal((C, H * D), dtype=f32) * f32(1.0 / np.sqrt(H * D))
    o = rng.standard_normal((B, H, T, D), dtype=f32)
    dq = rng.standard_normal((B, H, T, D), dtype=f32) * f32(0.01)
    dk = rng.standard_normal((B, H_kv, T, D), dtype=f32) * f32(0.01)
    dv = rng.standard_normal((B, H_kv, T, D), dtype=f32) * f32(0.01)
    dy = rng.standard_normal((B, T, C), dtype=f32) * f32(0.01)
    cu = draw_doc_lengths(rng, B, T, cfg.doc_lo, cfg.doc_hi) if packed else None
    x, w_qkv, w_o, o, dq, dk, dv, dy = (round_to_bf16(a) for a in (x, w_qkv, w_o, o, dq, dk, dv, dy))
    rc = rs = None
    if rope:
        rc, rs = rope_tables_f32(T, D, 10000.0)
    return ProjWorkload(cfg, x, w_qkv, w_o, o, dq, dk, dv, dy, rc, rs, cu)
