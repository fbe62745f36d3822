"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and compare them."""

from __future__ import annotations

import numpy as np

from oracle import attention_backward, attention_forward

# Relative Frobenius error bounds: bf16 storage with fp32 accumulation, and
# the float32 path.
TOL = {
    "bf16": {"o": 1e-2, "lse": 1e-4, "dq": 1e-2, "dk": 1e-2, "dv": 1e-2},
    "f32": {"o": 1e-5, "lse": 1e-5, "dq": 1e-5, "dk": 1e-5, "dv": 1e-5},
}

# Per-tile check: every 128-row tile of every compared slice must also meet
# TILE_FACTOR x the tensor's bound, its error taken relative to the larger of
# its own reference norm and TILE_FLOOR x the slice's RMS row norm scaled to
# the tile's row count. A tile's error has the expectation of the whole
# tensor's (the same roundings, on 128*D instead of T*D values); the factor
# leaves room for the tiles whose rows see few keys (the first rows of a
# causal head, short documents), and the floor keeps tiles whose reference
# is near zero (late keys' dk, dv) from dividing by almost nothing. A tile
# that is wrong as a whole fails by orders of magnitude; on an 8K head it
# would move the whole-tensor norm by only 1/8 of its own error.
TILE = 128
TILE_FACTOR = 2.0
TILE_FLOOR = 0.1


def rel_fro(got, ref) -> float:
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def tile_errors(got, ref) -> np.ndarray:
    """Relative error of every 128-row tile of every slice; got and ref are
    [n_slices, T] or [n_slices, T, D]."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    n, T = ref.shape[0], ref.shape[1]
    out = []
    for s in range(n):
        r_all = ref[s].reshape(T, -1)
        g_all = got[s].reshape(T, -1)
        rms_row = np.linalg.norm(r_all) / np.sqrt(T)
        for t0 in range(0, T, TILE):
            r = r_all[t0:t0 + TILE]
            g = g_all[t0:t0 + TILE]
            floor = TILE_FLOOR * rms_row * np.sqrt(r.shape[0])
            den = max(np.linalg.norm(r), floor)
            out.append(np.linalg.norm(g - r) / (den if den > 0 else 1.0))
    return np.asarray(out)


def oracle_outputs(w, heads=None) -> dict:
    o, lse = attention_forward(w.q, w.k, w.v, w.rope_cos, w.rope_sin, w.cu_seqlens, w.scale,
                               heads=heads)
    dq, dk, dv = attention_backward(w.q, w.k, w.v, w.do, w.rope_cos, w.rope_sin, w.cu_seqlens,
                                    w.scale, heads=heads)
    return {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}


def gpu_outputs(w, *, runner_cls=None) -> dict:
    from bwd_causal_sdpa_b200 import ATTN_OK
    from bwd_causal_sdpa_b200.runner import AttnRunner

    r = (runner_cls or AttnRunner).from_workload(w)
    r.forward()
    r.backward()
    st = r.status()
    assert st == ATTN_OK, f"device status {st}"
    return r.results()


def compare_arrays(got: dict, ref: dict, tol: dict, keys=None) -> dict:
    """Whole-tensor and per-tile errors of stacked slices ([n, T(, D)] per
    key); asserts both bounds and returns {key: error, key + "_tile": worst
    tile error}."""
    errs = {}
    bad = {}
    for key in (keys or list(ref)):
        g, r = got[key], ref[key]
        assert np.all(np.isfinite(g)), f"{key}: non-finite values"
        e = rel_fro(g, r)
        et = float(tile_errors(g, r).max())
        errs[key] = e
        errs[key + "_tile"] = et
        if not e <= tol[key]:
            bad[key] = (e, tol[key])
        if not et <= TILE_FACTOR * tol[key]:
            bad[key + "_tile"] = (et, TILE_FACTOR * tol[key])
    assert not bad, f"parity failed (error, bound): {bad}; all errors {errs}"
    return errs


def compare(w, got: dict, ref: dict, heads=None) -> dict:
    """Errors per tensor over the compared (b, h) query slices; asserts the
    bounds. dk and dv are compared on the key/value heads those slices read,
    which must come with every query head of their group (the oracle sums a
    shared head's gradient over the listed query heads only)."""
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    G = w.H // w.kv_heads
    kv_heads = sorted({(b, h // G) for b, h in heads})
    listed = set(heads)
    for b, hk in kv_heads:
        assert all((b, hk * G + g) in listed for g in range(G)), "incomplete query-head group"
    g_st, r_st = {}, {}
    for key in ("o", "lse", "dq", "dk", "dv"):
        pairs = kv_heads if key in ("dk", "dv") else heads
        g_st[key] = np.stack([got[key][b, h] for b, h in pairs])
        r_st[key] = np.stack([ref[key][b, h] for b, h in pairs])
    return compare_arrays(g_st, r_st, TOL[w.dtype], keys=("o", "lse", "dq", "dk", "dv"))
