"""Float64 oracle of the projections on either side of the attention.

TEST INFRASTRUCTURE (see the package docstring): never imported by the
library.

The attention layer of both training engines on the pages is
``x -> (q, k, v) = x W_qkv^T -> RoPE(q, k) -> SDPA -> o -> y = o W_o^T``
(ARK README, "Inference architecture (EKO)": RMSNorm, multi-head SDPA with
RoPE, then the FFN; its "Backward pass (AutoGrad)" lists the per-layer weight
gradients dwq, dwk, dwv, dwo. Forge README, "Architecture": ``Linear`` layers
and attention with GQA and interleaved-pair RoPE; "Benchmarks": the three
products of a linear layer, ``X W^T`` forward, ``dX = dY W`` and
``dW = dY^T X`` backward).

Conventions (readings where the pages are silent):
  * x is ``[B, T, C]``; W_qkv is ``[(H + 2 H_kv) D, C]``, its rows the q heads,
    then the k heads, then the v heads, each head's D features in order (the
    ``Linear`` convention ``y = x W^T`` with the three projections stacked).
  * q is written ``[B, H, T, D]``, k and v ``[B, H_kv, T, D]`` (the
    attention's layout).
  * RoPE, when tables are given, rotates q and k at each token's position in
    its document, exactly as the attention's own RoPE does; the attention is
    then called without tables.
  * W_o is ``[C, H D]`` and y ``[B, T, C]``; o is read in the attention's
    ``[B, H, T, D]`` layout, feature index h * D + d.
  * The backward takes the gradients with respect to the forward's outputs
    (for q, k: the rotated ones when the forward rotated) and returns dx and
    the weight gradient for the loss sum(outputs * gradients).
Every function upcasts its inputs exactly to float64 and rounds nothing.
"""

from typing import Optional, Tuple

import numpy as np

from .attention import doc_layout, rope_rotate, rope_rotate_inverse


def _f64(*arrs):
    return tuple(np.asarray(a, dtype=np.float64) for a in arrs)


def _split_heads(y: np.ndarray, B: int, T: int, heads: int, D: int) -> np.ndarray:
    """[B, T, heads * D] -> [B, heads, T, D]."""
    return y.reshape(B, T, heads, D).transpose(0, 2, 1, 3)


def _merge_heads(t: np.ndarray) -> np.ndarray:
    """[B, heads, T, D] -> [B, T, heads * D] (feature index h * D + d)."""
    B, heads, T, D = t.shape
    return t.transpose(0, 2, 1, 3).reshape(B, T, heads * D)


def qkv_projection(x, w_qkv, H: int, H_kv: int, D: int, rope_cos=None, rope_sin=None,
                   cu_seqlens: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """q, k, v = heads of x W_qkv^T; q and k rotated when tables are given."""
    x, w = _f64(x, w_qkv)
    B, T, C = x.shape
    if w.shape != ((H + 2 * H_kv) * D, C):
        raise ValueError("w_qkv must be [(H + 2 H_kv) D, C]")
    y = x @ w.T
    q = _split_heads(y[:, :, :H * D], B, T, H, D).copy()
    k = _split_heads(y[:, :, H * D:(H + H_kv) * D], B, T, H_kv, D).copy()
    v = _split_heads(y[:, :, (H + H_kv) * D:], B, T, H_kv, D).copy()
    if rope_cos is not None:
        cos, sin = _f64(rope_cos, rope_sin)
        pos, _ = doc_layout(B, T, cu_seqlens)
        for b in range(B):
            for h in range(H):
                q[b, h] = rope_rotate(q[b, h], cos, sin, pos[b])
            for h in range(H_kv):
                k[b, h] = rope_rotate(k[b, h], cos, sin, pos[b])
    return q, k, v


def qkv_projection_backward(dq, dk, dv, x, w_qkv, rope_cos=None, rope_sin=None,
                            cu_seqlens: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """dx = dY W_qkv and dW_qkv = dY^T x, dY the [B, T, (H + 2 H_kv) D]
    gradient of the un-rotated projection (R^T applied to dq, dk first when
    the forward rotated)."""
    dq, dk, dv, x, w = _f64(dq, dk, dv, x, w_qkv)
    B, H, T, D = dq.shape
    H_kv = dk.shape[1]
    C = x.shape[2]
    if rope_cos is not None:
        cos, sin = _f64(rope_cos, rope_sin)
        pos, _ = doc_layout(B, T, cu_seqlens)
        dq = dq.copy()
        dk = dk.copy()
        for b in range(B):
            for h in range(H):
                dq[b, h] = rope_rotate_inverse(dq[b, h], cos, sin, pos[b])
            for h in range(H_kv):
                dk[b, h] = rope_rotate_inverse(dk[b, h], cos, sin, pos[b])
    dy = np.concatenate([_merge_heads(dq), _merge_heads(dk), _merge_heads(dv)], axis=2)
    dx = dy @ w
    dw = dy.reshape(B * T, -1).T @ x.reshape(B * T, C)
    return dx, dw


def out_projection(o, w_o) -> np.ndarray:
    """y = o W_o^T with o read as [B, T, H D]."""
    o, w = _f64(o, w_o)
    return _merge_heads(o) @ w.T


def out_projection_backward(dy, o, w_o) -> Tuple[np.ndarray, np.ndarray]:
    """d_o = dy W_o (back in [B, H, T, D]) and dW_o = dy^T o."""
    dy, o, w = _f64(dy, o, w_o)
    B, H, T, D = o.shape
    C = dy.shape[2]
    d_o = _split_heads(dy @ w, B, T, H, D).copy()
    dw = dy.reshape(B * T, C).T @ _merge_heads(o).reshape(B * T, H * D)
    return d_o, dw
