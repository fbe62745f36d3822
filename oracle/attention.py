"""float64 oracle for causal multi-head attention with RoPE and packed documents.

TEST INFRASTRUCTURE: imported only by tests/, __graft_entry__.smoke() and the
cpu_baseline leg of bench.py. Dense and deliberately unoptimised: the full
score matrix of one (batch, head) slice is materialised, masked, normalised
with a three-pass softmax and multiplied out; the backward is the analytic
gradient written term by term. No blocking, no online softmax, no fusion.

Sources (page title, section):
- ARK README, "Inference architecture (EKO)" and "Accelerated forward pass":
  multi-head SDPA with a causal mask fused into it, RoPE from precomputed
  sin/cos tables, gradients of the attention produced by autograd.
- ARK README, asm/kern.s entry: softmax in three passes (max, sum of
  exponentials, normalise), the underflow-safe form used below.
- Forge README, "Architecture", Model line: RoPE applied to interleaved pairs
  (2i, 2i+1); attention behind an interface that also serves training.
- Forge README, "What this is" and "Verified": flash attention forward and
  backward validated against a CPU reference and by numerical gradient checks.
- Cort33x, "Preserving context in the data": short documents packed into one
  training window with separators; here every document attends only to itself
  (within-document causal mask) and its RoPE positions restart at 0.

Conventions (the plainest reading where the pages are silent):
- tensors are [B, H, T, D] (D fastest); lse is [B, H, T];
- lse is the natural log of the sum of exp(scale * q_r . k_r) over allowed keys;
- a token attends to itself (j <= i), so no row is empty;
- cu_seqlens indexes the flattened B*T token axis, starts at 0, ends at B*T and
  contains every row boundary r*T (documents never cross rows);
- the backward returns gradients with respect to the un-rotated q and k;
- grouped-query attention (Forge README, "Architecture": attention with GQA
  and RoPE): k and v may have H_kv heads with H_kv dividing H; query head h
  reads key/value head h // (H / H_kv), and the gradient of a shared key/value
  head is the sum over the query heads that read it.
"""

from __future__ import annotations

from typing import Iterable, Optional, Sequence, Tuple

import numpy as np


# ----------------------------------------------------------------------------
# RoPE: a rotation of each interleaved pair (x[2i], x[2i+1]) by pos * theta_i
# ----------------------------------------------------------------------------

def rope_angles_f64(T: int, D: int, theta: float = 10000.0) -> Tuple[np.ndarray, np.ndarray]:
    """The oracle's own tables: cos and sin of p * theta^(-2i/D), float64, [T, D/2].

    (ARK README: RoPE "with precomputed sin/cos tables"; the frequency ladder
    theta^(-2i/D) is the RoFormer one the ARK README lists among its sources.)
    """
    i = np.arange(D // 2, dtype=np.float64)
    freq = np.power(float(theta), -2.0 * i / float(D))
    angle = np.outer(np.arange(T, dtype=np.float64), freq)
    return np.cos(angle), np.sin(angle)


def rope_rotate(x: np.ndarray, cos: np.ndarray, sin: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """R(pos) x for x of shape [T, D]: each pair (x0, x1) = (x[2i], x[2i+1])
    becomes (x0*c - x1*s, x0*s + x1*c) with c, s the table entries at
    (pos[t], i). (Forge README, Architecture: RoPE on interleaved pairs.)"""
    c = cos[pos]
    s = sin[pos]
    x0 = x[:, 0::2]
    x1 = x[:, 1::2]
    y = np.empty_like(x)
    y[:, 0::2] = x0 * c - x1 * s
    y[:, 1::2] = x0 * s + x1 * c
    return y


def rope_rotate_inverse(g: np.ndarray, cos: np.ndarray, sin: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """R(pos)^T g: the transpose rotation, which carries a gradient taken with
    respect to the rotated vector back to the un-rotated input."""
    c = cos[pos]
    s = sin[pos]
    g0 = g[:, 0::2]
    g1 = g[:, 1::2]
    y = np.empty_like(g)
    y[:, 0::2] = g0 * c + g1 * s
    y[:, 1::2] = -g0 * s + g1 * c
    return y


# ----------------------------------------------------------------------------
# Packed documents
# ----------------------------------------------------------------------------

def doc_layout(B: int, T: int, cu_seqlens: Optional[np.ndarray]) -> Tuple[np.ndarray, np.ndarray]:
    """Per token of each row: its RoPE position and the row-local index where
    its document starts. Without cu_seqlens every row is one document.

    (Cort33x, "Preserving context in the data": short documents packed into a
    window; positions restart and attention stays inside each document.)
    """
    pos = np.tile(np.arange(T, dtype=np.int64), (B, 1))
    start = np.zeros((B, T), dtype=np.int64)
    if cu_seqlens is None:
        return pos, start
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    if cu[0] != 0 or cu[-1] != B * T or np.any(np.diff(cu) <= 0):
        raise ValueError("cu_seqlens must rise strictly from 0 to B*T")
    for r in range(B + 1):
        if r * T not in set(cu.tolist()):
            raise ValueError("cu_seqlens must contain every row boundary r*T")
    for a, e in zip(cu[:-1], cu[1:]):
        b = int(a // T)
        lo, hi = int(a - b * T), int(e - b * T)
        pos[b, lo:hi] = np.arange(hi - lo)
        start[b, lo:hi] = lo
    return pos, start


def allowed_keys(doc_start: np.ndarray) -> np.ndarray:
    """[T, T] boolean: query i may attend key j iff j <= i and j lies in i's
    document (j >= doc_start[i]). (ARK README: causal mask fused into SDPA.)"""
    T = doc_start.shape[0]
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    return (j <= i) & (j >= doc_start[:, None])


# ----------------------------------------------------------------------------
# One (batch, head) slice
# ----------------------------------------------------------------------------

def _softmax_three_pass(S: np.ndarray, allowed: np.ndarray):
    """Row softmax over allowed entries in three passes (ARK README, kern.s:
    max, then sum of exp(S - max), then divide). Returns P and the natural-log
    sum-exp per row."""
    Sm = np.where(allowed, S, -np.inf)
    m = Sm.max(axis=1, keepdims=True)                 # pass 1
    e = np.exp(Sm - m)                                # masked entries -> 0
    l = e.sum(axis=1, keepdims=True)                  # pass 2
    P = e / l                                         # pass 3
    lse = (m + np.log(l))[:, 0]
    return P, lse


def forward_head(q, k, v, cos, sin, pos, doc_start, scale):
    """Forward of one slice; q, k, v are [T, D] float64.

    cos/sin None means no RoPE. Returns a dict with o [T, D], lse [T] and the
    intermediates (q_r, k_r, S, P) the backward and the tests reuse.
    """
    if cos is not None:
        qr = rope_rotate(q, cos, sin, pos)
        kr = rope_rotate(k, cos, sin, pos)
    else:
        qr, kr = q, k
    allowed = allowed_keys(doc_start)
    S = scale * (qr @ kr.T)
    P, lse = _softmax_three_pass(S, allowed)
    o = P @ v
    return {"o": o, "lse": lse, "qr": qr, "kr": kr, "S": S, "P": P, "allowed": allowed}


def backward_head(q, k, v, do, cos, sin, pos, doc_start, scale, fwd=None):
    """Analytic backward of L = sum(o * do) for one slice (float64).

    Delta_i = sum_d do[i,d] * o[i,d]; dP = do v^T; dS = P * (dP - Delta);
    dv = P^T do; dq_r = scale * dS k_r; dk_r = scale * dS^T q_r; and, with RoPE,
    dq = R(pos)^T dq_r, dk = R(pos)^T dk_r.
    """
    f = forward_head(q, k, v, cos, sin, pos, doc_start, scale) if fwd is None else fwd
    P, o, qr, kr = f["P"], f["o"], f["qr"], f["kr"]
    delta = (do * o).sum(axis=1)
    dP = do @ v.T
    dS = P * (dP - delta[:, None])
    dv = P.T @ do
    dqr = scale * (dS @ kr)
    dkr = scale * (dS.T @ qr)
    if cos is not None:
        dq = rope_rotate_inverse(dqr, cos, sin, pos)
        dk = rope_rotate_inverse(dkr, cos, sin, pos)
    else:
        dq, dk = dqr, dkr
    return {"dq": dq, "dk": dk, "dv": dv, "dS": dS, "delta": delta, "fwd": f}


# ----------------------------------------------------------------------------
# Whole tensors [B, H, T, D]
# ----------------------------------------------------------------------------

def _tables(rope_cos, rope_sin):
    if rope_cos is None:
        return None, None
    return (np.asarray(rope_cos, dtype=np.float64), np.asarray(rope_sin, dtype=np.float64))


def _slices(B: int, H: int, heads: Optional[Iterable[Tuple[int, int]]]) -> Sequence[Tuple[int, int]]:
    if heads is None:
        return [(b, h) for b in range(B) for h in range(H)]
    return list(heads)


def _kv_head(h: int, H: int, H_kv: int) -> int:
    if H % H_kv:
        raise ValueError("the number of query heads must be a multiple of the key/value heads")
    return h // (H // H_kv)


def attention_forward(q, k, v, rope_cos, rope_sin, cu_seqlens, scale, heads=None):
    """o [B,H,T,D] and lse [B,H,T] in float64. Inputs are upcast exactly from
    their float32/bf16 storage; k, v may have fewer heads than q (grouped-query
    attention). ``heads`` optionally restricts the work to a list of (b, h)
    query slices (the other entries are left NaN)."""
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    B, H, T, D = q.shape
    H_kv = k.shape[1]
    cos, sin = _tables(rope_cos, rope_sin)
    pos, start = doc_layout(B, T, cu_seqlens)
    o = np.full((B, H, T, D), np.nan)
    lse = np.full((B, H, T), np.nan)
    for b, h in _slices(B, H, heads):
        hk = _kv_head(h, H, H_kv)
        f = forward_head(q[b, h], k[b, hk], v[b, hk], cos, sin, pos[b], start[b], scale)
        o[b, h] = f["o"]
        lse[b, h] = f["lse"]
    return o, lse


def attention_backward(q, k, v, do, rope_cos, rope_sin, cu_seqlens, scale, heads=None):
    """dq [B,H,T,D] and dk, dv [B,H_kv,T,D] in float64 for the loss
    L = sum(o * do), with o the exact forward of the same inputs. With
    ``heads`` (a list of (b, h) query slices) only those slices' contributions
    are computed: dq for them, and dk, dv summed over them for the key/value
    heads they read (entries no listed slice reads are left NaN)."""
    q, k, v, do = (np.asarray(a, dtype=np.float64) for a in (q, k, v, do))
    B, H, T, D = q.shape
    H_kv = k.shape[1]
    cos, sin = _tables(rope_cos, rope_sin)
    pos, start = doc_layout(B, T, cu_seqlens)
    dq = np.full((B, H, T, D), np.nan)
    dk = np.full((B, H_kv, T, D), np.nan)
    dv = np.full((B, H_kv, T, D), np.nan)
    for b, h in _slices(B, H, heads):
        hk = _kv_head(h, H, H_kv)
        g = backward_head(q[b, h], k[b, hk], v[b, hk], do[b, h], cos, sin, pos[b], start[b], scale)
        dq[b, h] = g["dq"]
        if np.isnan(dk[b, hk, 0, 0]):
            dk[b, hk] = 0.0
            dv[b, hk] = 0.0
        dk[b, hk] += g["dk"]
        dv[b, hk] += g["dv"]
    return dq, dk, dv
