"""Seeded decode workloads: one new token per sequence against a key/value
cache (no attention arithmetic lives here).

Draw order from ``numpy.random.default_rng(seed)``: the cache lengths
(``integers(len_min, T_max + 1)`` per batch row), then float32 standard
normals scaled by their standard deviations: q [B, H, D], the cached keys
[B, H_kv, T_max, D], the cached values [B, H_kv, T_max, D]. The cached keys
stand for keys already rotated by their positions: a rotation of a vector of
independent standard normals is again one, so they are drawn as such and no
rotation is done here. bf16 workloads round every tensor to bf16 (RNE).
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import numpy as np

from .generate import rope_tables_f32, round_to_bf16


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    dtype: str      # "bf16" or "f32"
    B: int
    H: int
    H_kv: int
    T_max: int      # cache capacity per sequence
    D: int
    len_min: int    # cache lengths drawn uniformly from [len_min, T_max]
    rope: bool
    theta: float
    qk_std: float
    v_std: float
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


DECODE_CONFIGS = [
    # generation with a long grouped-query cache (32 query heads on 8 cached heads)
    DecodeConfig("decode_8k_gqa", "bf16", 8, 32, 8, 8192, 128, 4096, True, 10000.0, 1.0, 1.0, 20),
    # generation on the 237M decoder layer shape (16 heads of 64, 1K context)
    DecodeConfig("decode_237m", "bf16", 16, 16, 16, 1024, 64, 512, True, 10000.0, 1.5, 1.0, 21),
]


def decode_config_by_name(name: str) -> DecodeConfig:
    for c in DECODE_CONFIGS:
        if c.name == name:
            return c
    raise KeyError(f"unknown decode workload {name!r}; known: {[c.name for c in DECODE_CONFIGS]}")


@dataclass
class DecodeWorkload:
    cfg: DecodeConfig
    B: int
    H: int
    H_kv: int
    T_max: int
    D: int
    q: np.ndarray
    k_cache: np.ndarray
    v_cache: np.ndarray
    cache_lens: np.ndarray
    rope_cos: Optional[np.ndarray]
    rope_sin: Optional[np.ndarray]
    scale: float

    @property
    def dtype(self) -> str:
        return self.cfg.dtype

    def cache_bytes_read(self) -> int:
        """Bytes of keys and values one decode step must read: 2 * H_kv * D
        values of the storage type per cached token of every sequence."""
        elem = 2 if self.dtype == "bf16" else 4
        return int(2 * self.H_kv * self.D * elem * int(self.cache_lens.astype(np.int64).sum()))


def make_decode_workload(cfg: DecodeConfig, *, B: Optional[int] = None, H: Optional[int] = None,
                         H_kv: Optional[int] = None, T_max: Optional[int] = None,
                         D: Optional[int] = None, len_min: Optional[int] = None,
                         seed: Optional[int] = None, rope: Optional[bool] = None,
                         dtype: Optional[str] = None) -> DecodeWorkload:
    B = cfg.B if B is None else B
    H = cfg.H if H is None else H
    H_kv = cfg.H_kv if H_kv is None else H_kv
    T_max = cfg.T_max if T_max is None else T_max
    D = cfg.D if D is None else D
    len_min = cfg.len_min if len_min is None else len_min
    seed = cfg.seed if seed is None else seed
    rope = cfg.rope if rope is None else rope
    dtype = cfg.dtype if dtype is None else dtype
    if H % H_kv:
        raise ValueError("H_kv must divide H")
    len_min = max(1, min(len_min, T_max))
    rng = np.random.default_rng(seed)
    lens = rng.integers(len_min, T_max + 1, size=B).astype(np.int32)
    q = rng.standard_normal((B, H, D), dtype=np.float32) * np.float32(cfg.qk_std)
    kc = rng.standard_normal((B, H_kv, T_max, D), dtype=np.float32) * np.float32(cfg.qk_std)
    vc = rng.standard_normal((B, H_kv, T_max, D), dtype=np.float32) * np.float32(cfg.v_std)
    if dtype == "bf16":
        q, kc, vc = (round_to_bf16(a) for a in (q, kc, vc))
    rc = rs = None
    if rope:
        rc, rs = rope_tables_f32(T_max, D, cfg.theta)
    cfg_used = cfg if dtype == cfg.dtype else DecodeConfig(**{**cfg.__dict__, "dtype": dtype})
    return DecodeWorkload(cfg_used, B, H, H_kv, T_max, D, q, kc, vc, lens, rc, rs,
                          1.0 / float(np.sqrt(D)))
