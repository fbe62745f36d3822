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


def rel_fro(got, ref) -> float:
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


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
    tol = TOL[w.dtype]
    errs = {}
    for key in ("o", "lse", "dq", "dk", "dv"):
        pairs = kv_heads if key in ("dk", "dv") else heads
        g = np.stack([got[key][b, h] for b, h in pairs])
        r = np.stack([ref[key][b, h] for b, h in pairs])
        assert np.all(np.isfinite(g)), f"{key}: non-finite values"
        errs[key] = rel_fro(g, r)
    bad = {k: (e, tol[k]) for k, e in errs.items() if not e <= tol[k]}
    assert not bad, f"parity failed (error, bound): {bad}; all errors {errs}"
    return errs
