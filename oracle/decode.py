"""float64 oracle for decode attention: one new token per sequence against a
key/value cache.

TEST INFRASTRUCTURE (imported only by tests/ and bench.py's cpu_baseline
leg, like the rest of ``oracle``). Dense and unoptimised: for each (batch,
head) the scores of the new query against every cached key are formed, then
a three-pass softmax and the weighted sum of the cached values.

Sources (page title, section):
- Forge README, "Roadmap": a KV cache for generation, on the same attention
  module the training path uses ("Architecture": attention with GQA + RoPE).
- ARK README, "Inference architecture (EKO)": generation with RoPE from
  precomputed sin/cos tables.

Reading (the pages name the cache but give no interface; the plainest one):
- the cache holds, per batch row b, cache_lens[b] tokens at positions
  0 .. cache_lens[b]-1, the newest token's own key and value included; keys
  are stored already rotated by their positions (as the forward rotates k);
- the new token's query sits at position cache_lens[b]-1, is rotated there,
  and attends to every cached token (causality holds by construction);
- with H_kv key/value heads, query head h reads cache head h // (H / H_kv).
The result is therefore the last row of the training forward on the whole
sequence, which is what the pins check.
"""

from __future__ import annotations

import numpy as np

from .attention import rope_rotate


def decode_forward(q, k_cache, v_cache, cache_lens, rope_cos, rope_sin, scale, heads=None):
    """o [B, H, D] and lse [B, H] (natural log) in float64.

    q [B, H, D] (un-rotated); k_cache, v_cache [B, H_kv, T_max, D] (keys
    rotated); cache_lens [B] with 1 <= cache_lens[b] <= T_max. ``heads``
    optionally restricts the work to a list of (b, h) slices (others NaN).
    """
    q, k_cache, v_cache = (np.asarray(a, dtype=np.float64) for a in (q, k_cache, v_cache))
    B, H, D = q.shape
    H_kv, T_max = k_cache.shape[1], k_cache.shape[2]
    if H % H_kv:
        raise ValueError("the number of query heads must be a multiple of the key/value heads")
    G = H // H_kv
    lens = np.asarray(cache_lens, dtype=np.int64)
    if lens.shape != (B,) or np.any(lens < 1) or np.any(lens > T_max):
        raise ValueError("cache_lens must hold B lengths in [1, T_max]")
    cos = None if rope_cos is None else np.asarray(rope_cos, dtype=np.float64)
    sin = None if rope_sin is None else np.asarray(rope_sin, dtype=np.float64)
    o = np.full((B, H, D), np.nan)
    lse = np.full((B, H), np.nan)
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    for b, h in pairs:
        L = int(lens[b])
        qv = q[b, h][None, :]
        if cos is not None:
            qv = rope_rotate(qv, cos, sin, np.array([L - 1]))
        k = k_cache[b, h // G, :L]
        v = v_cache[b, h // G, :L]
        s = scale * (k @ qv[0])               # scores against every cached key
        m = s.max()                           # pass 1
        e = np.exp(s - m)
        l = e.sum()                           # pass 2
        o[b, h] = (e / l) @ v                 # pass 3, weighted sum
        lse[b, h] = m + np.log(l)
    return o, lse
