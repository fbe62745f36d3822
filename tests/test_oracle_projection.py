"""Pins of the projection oracle (CPU only).

Each check ties ``oracle.projection`` to something other than its own
formulas: explicit index sums written as loops, the attention oracle's RoPE
(rotating inside the projection must equal rotating inside the attention),
identity weights that reduce the projections to a relabelling of the input,
and central finite differences of the loss sum(outputs * gradients) for every
backward product.
"""

import itertools

import numpy as np
import pytest

from oracle import (attention_forward, out_projection, out_projection_backward, qkv_projection,
                    qkv_projection_backward)
from workloads import rope_tables_f32


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_qkv_projection_matches_index_sums():
    rng = np.random.default_rng(0)
    B, T, C, H, H_kv, D = 2, 3, 5, 2, 1, 4
    x = _rand(rng, B, T, C)
    w = _rand(rng, (H + 2 * H_kv) * D, C)
    q, k, v = qkv_projection(x, w, H, H_kv, D)
    for b, t, d in itertools.product(range(B), range(T), range(D)):
        for h in range(H):
            ref = sum(x[b, t, c] * w[h * D + d, c] for c in range(C))
            assert q[b, h, t, d] == pytest.approx(ref, rel=1e-12, abs=1e-12)
        for h in range(H_kv):
            rk = sum(x[b, t, c] * w[(H + h) * D + d, c] for c in range(C))
            rv = sum(x[b, t, c] * w[(H + H_kv + h) * D + d, c] for c in range(C))
            assert k[b, h, t, d] == pytest.approx(rk, rel=1e-12, abs=1e-12)
            assert v[b, h, t, d] == pytest.approx(rv, rel=1e-12, abs=1e-12)


def test_out_projection_matches_index_sums():
    rng = np.random.default_rng(1)
    B, H, T, D, C = 2, 3, 2, 4, 5
    o = _rand(rng, B, H, T, D)
    w = _rand(rng, C, H * D)
    y = out_projection(o, w)
    for b, t, c in itertools.product(range(B), range(T), range(C)):
        ref = sum(o[b, h, t, d] * w[c, h * D + d] for h in range(H) for d in range(D))
        assert y[b, t, c] == pytest.approx(ref, rel=1e-12, abs=1e-12)


def test_identity_weights_relabel_the_input():
    rng = np.random.default_rng(2)
    B, T, H, D = 1, 4, 2, 4
    C = H * D
    x = _rand(rng, B, T, C)
    eye = np.eye(C)
    q, k, v = qkv_projection(x, np.concatenate([eye, eye, eye]), H, H, D)
    heads = x.reshape(B, T, H, D).transpose(0, 2, 1, 3)
    assert np.array_equal(q, heads) and np.array_equal(k, heads) and np.array_equal(v, heads)
    assert np.array_equal(out_projection(heads, eye), x)


@pytest.mark.parametrize("packed", [False, True])
def test_rope_in_projection_equals_rope_in_attention(packed):
    rng = np.random.default_rng(3)
    B, T, C, H, H_kv, D = 2, 12, 6, 2, 1, 8
    x = _rand(rng, B, T, C)
    w = _rand(rng, (H + 2 * H_kv) * D, C)
    cos, sin = rope_tables_f32(T, D, 10000.0)
    cu = np.array([0, 5, 12, 15, 24], dtype=np.int32) if packed else None
    q_r, k_r, v_r = qkv_projection(x, w, H, H_kv, D, cos, sin, cu)
    q, k, v = qkv_projection(x, w, H, H_kv, D)
    assert np.array_equal(v, v_r)
    scale = 1.0 / np.sqrt(D)
    o1, l1 = attention_forward(q_r, k_r, v_r, None, None, cu, scale)
    o2, l2 = attention_forward(q, k, v, cos, sin, cu, scale)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=1e-12, atol=1e-12)


def _central(f, arr, idx, h=1e-3):
    old = arr[idx]
    arr[idx] = old + h
    fp = f()
    arr[idx] = old - h
    fm = f()
    arr[idx] = old
    return (fp - fm) / (2 * h)


@pytest.mark.parametrize("rope,packed", [(False, False), (True, False), (True, True)])
def test_qkv_backward_matches_finite_differences(rope, packed):
    rng = np.random.default_rng(4)
    B, T, C, H, H_kv, D = 2, 6, 5, 2, 1, 4
    x = _rand(rng, B, T, C)
    w = _rand(rng, (H + 2 * H_kv) * D, C)
    gq, gk, gv = _rand(rng, B, H, T, D), _rand(rng, B, H_kv, T, D), _rand(rng, B, H_kv, T, D)
    cos, sin = rope_tables_f32(T, D, 10000.0) if rope else (None, None)
    cu = np.array([0, 2, 6, 9, 12], dtype=np.int32) if packed else None

    def loss():
        q, k, v = qkv_projection(x, w, H, H_kv, D, cos, sin, cu)
        return float(np.sum(q * gq) + np.sum(k * gk) + np.sum(v * gv))

    dx, dw = qkv_projection_backward(gq, gk, gv, x, w, cos, sin, cu)
    for idx in [(0, 0, 0), (1, 5, 4), (0, 3, 2), (1, 2, 1)]:
        assert dx[idx] == pytest.approx(_central(loss, x, idx), rel=1e-8, abs=1e-9)
    for idx in [(0, 0), (3, 4), (H * D, 1), ((H + H_kv) * D + 2, 3), (w.shape[0] - 1, 0)]:
        assert dw[idx] == pytest.approx(_central(loss, w, idx), rel=1e-8, abs=1e-9)


def test_out_backward_matches_finite_differences():
    rng = np.random.default_rng(5)
    B, H, T, D, C = 2, 2, 3, 4, 5
    o = _rand(rng, B, H, T, D)
    w = _rand(rng, C, H * D)
    gy = _rand(rng, B, T, C)

    def loss():
        return float(np.sum(out_projection(o, w) * gy))

    d_o, dw = out_projection_backward(gy, o, w)
    for idx in [(0, 0, 0, 0), (1, 1, 2, 3), (0, 1, 1, 2)]:
        assert d_o[idx] == pytest.approx(_central(loss, o, idx), rel=1e-8, abs=1e-9)
    for idx in [(0, 0), (4, 7), (2, 5)]:
        assert dw[idx] == pytest.approx(_central(loss, w, idx), rel=1e-8, abs=1e-9)


# --------------------------------------------------------------------------
# Planted mistakes: every mutant of the projection oracle must fail a pin
# --------------------------------------------------------------------------

import oracle.projection as P  # noqa: E402


def _pins_pass():
    checks = [test_qkv_projection_matches_index_sums,
              test_out_projection_matches_index_sums,
              test_identity_weights_relabel_the_input,
              lambda: test_rope_in_projection_equals_rope_in_attention(True),
              lambda: test_qkv_backward_matches_finite_differences(True, True),
              lambda: test_qkv_backward_matches_finite_differences(False, False),
              test_out_backward_matches_finite_differences]
    for c in checks:
        try:
            c()
        except (AssertionError, ValueError, IndexError):
            return False
    return True


_orig_split, _orig_merge = P._split_heads, P._merge_heads
_orig_qkv, _orig_rot, _orig_inv = P.qkv_projection, P.rope_rotate, P.rope_rotate_inverse


def _mut_split_d_major(y, B, T, heads, D):
    # features read as d-major (d * heads + h) instead of head-major
    return y.reshape(B, T, D, heads).transpose(0, 3, 1, 2)


def _mut_merge_d_major(t):
    B, heads, T, D = t.shape
    return t.transpose(0, 2, 3, 1).reshape(B, T, heads * D)


def _mut_k_v_swapped(x, w_qkv, H, H_kv, D, rope_cos=None, rope_sin=None, cu_seqlens=None):
    q, k, v = _orig_qkv(x, w_qkv, H, H_kv, D, rope_cos, rope_sin, cu_seqlens)
    return q, v, k


def _mut_backward_no_inverse(g, cos, sin, pos):
    return g  # the gradient of the rotated q, k used as if un-rotated


MUTANTS = {
    "heads_read_d_major": ("_split_heads", _mut_split_d_major),
    "heads_merged_d_major": ("_merge_heads", _mut_merge_d_major),
    "k_and_v_swapped": ("qkv_projection", _mut_k_v_swapped),
    "backward_skips_inverse_rope": ("rope_rotate_inverse", _mut_backward_no_inverse),
    "backward_rotates_forward": ("rope_rotate_inverse", lambda g, c, s, p: _orig_rot(g, c, s, p)),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_is_caught(mutant, monkeypatch):
    assert _pins_pass()
    attr, fn = MUTANTS[mutant]
    monkeypatch.setattr(P, attr, fn)
    if attr == "qkv_projection":  # the pins call it through this module's own import
        monkeypatch.setitem(globals(), "qkv_projection", fn)
    assert not _pins_pass(), f"no pin caught the planted mistake {mutant}"
