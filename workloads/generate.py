"""Seeded input generation (no attention arithmetic lives here).

Draw order for one workload, from ``numpy.random.default_rng(seed)``:
q, k, v, dO as float32 standard normals of shape [B, H, T, D] (each scaled by
its standard deviation), then, for packed documents, document lengths drawn
with ``integers(doc_min, doc_max + 1)`` row by row until the row is full, the
last one truncated. bf16 workloads round every tensor to bf16
(round-to-nearest-even) on the host; the rounded values are the inputs both
sides see.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from .configs import Config


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32.

    Implemented on the bit pattern: add 0x7FFF plus the lowest kept bit, then
    clear the 16 dropped bits. Inputs here are finite normals, so no NaN path.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of float32 values that are already bf16-representable."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def rope_tables_f32(T: int, D: int, theta: float):
    """Caller-side RoPE tables, as a training engine would precompute them.

    cos[p, i] = cos(p * theta^(-2i/D)) and sin[p, i] likewise, for positions
    p in [0, T) and pair index i in [0, D/2); evaluated in float64 and rounded
    to float32 once. Shape [T, D/2] each, row p is position p.
    """
    i = np.arange(D // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / D)
    ang = np.arange(T, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def draw_doc_lengths(rng: np.random.Generator, B: int, T: int, lo: int, hi: int) -> np.ndarray:
    """cu_seqlens over the flattened B*T token axis: every row is filled with
    documents of length Uniform[lo, hi] (the last one truncated to the row end),
    so every row boundary r*T is present and the final entry is B*T."""
    cu = [0]
    for b in range(B):
        filled = 0
        while filled < T:
            n = int(rng.integers(lo, hi + 1))
            n = min(n, T - filled)
            filled += n
            cu.append(b * T + filled)
    return np.asarray(cu, dtype=np.int32)


@dataclass
class Workload:
    cfg: Config
    B: int
    H: int
    T: int
    D: int
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    do: np.ndarray
    cu_seqlens: Optional[np.ndarray]
    rope_cos: Optional[np.ndarray]
    rope_sin: Optional[np.ndarray]
    scale: float
    H_kv: Optional[int] = None  # key/value heads (grouped-query attention); None = H

    @property
    def kv_heads(self) -> int:
        return self.H if self.H_kv is None else self.H_kv

    @property
    def dtype(self) -> str:
        return self.cfg.dtype

    def doc_lengths(self) -> list:
        if self.cu_seqlens is None:
            return [self.T] * self.B
        return list(np.diff(self.cu_seqlens.astype(np.int64)))

    def algorithmic_flops(self) -> float:
        """7 * H * D * sum over documents of L^2 (the nominal convention with the
        masked work removed; equals 7*B*H*T^2*D when every row is one document)."""
        L = np.asarray(self.doc_lengths(), dtype=np.float64)
        return 7.0 * self.H * self.D * float((L * L).sum())


def make_workload(cfg: Config, *, B: Optional[int] = None, H: Optional[int] = None,
                  T: Optional[int] = None, D: Optional[int] = None,
                  seed: Optional[int] = None, varlen: Optional[bool] = None,
                  rope: Optional[bool] = None, doc_min: Optional[int] = None,
                  doc_max: Optional[int] = None, H_kv: Optional[int] = None) -> Workload:
    """Draw one workload. Keyword overrides give smaller parity cases with the
    same value distributions and structure as ``cfg``; ``H_kv`` (dividing H)
    draws k and v with that many heads for grouped-query attention."""
    B = cfg.B if B is None else B
    H = cfg.H if H is None else H
    T = cfg.T if T is None else T
    D = cfg.D if D is None else D
    seed = cfg.seed if seed is None else seed
    varlen = cfg.varlen if varlen is None else varlen
    rope = cfg.rope if rope is None else rope
    doc_min = cfg.doc_min if doc_min is None else doc_min
    doc_max = cfg.doc_max if doc_max is None else doc_max

    if H_kv is not None and (H_kv <= 0 or H % H_kv):
        raise ValueError("H_kv must divide H")
    rng = np.random.default_rng(seed)
    shape = (B, H, T, D)
    kv_shape = shape if H_kv is None else (B, H_kv, T, D)
    q = rng.standard_normal(shape, dtype=np.float32) * np.float32(cfg.qk_std)
    k = rng.standard_normal(kv_shape, dtype=np.float32) * np.float32(cfg.qk_std)
    v = rng.standard_normal(kv_shape, dtype=np.float32) * np.float32(cfg.v_std)
    do = rng.standard_normal(shape, dtype=np.float32) * np.float32(cfg.do_std)
    cu = draw_doc_lengths(rng, B, T, doc_min, doc_max) if varlen else None
    if cfg.dtype == "bf16":
        q, k, v, do = (round_to_bf16(a) for a in (q, k, v, do))
    if rope:
        rc, rs = rope_tables_f32(T, D, cfg.theta)
    else:
        rc = rs = None
    return Workload(cfg, B, H, T, D, q, k, v, do, cu, rc, rs, 1.0 / float(np.sqrt(D)), H_kv)
