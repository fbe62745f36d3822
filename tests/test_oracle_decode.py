"""Pins of the decode oracle (CPU): the last row of the training forward on
the whole sequence, a closed form, invariants and the grouped-head mapping.
A planted mistake (the query rotated at the wrong position) must fail."""

import numpy as np
import pytest

from oracle import attention_forward, decode_forward, rope_angles_f64, rope_rotate


def _sequence(rng, B, H, H_kv, T, D):
    q = rng.standard_normal((B, H, T, D))
    k = rng.standard_normal((B, H_kv, T, D))
    v = rng.standard_normal((B, H_kv, T, D))
    return q, k, v


def _rotated_cache(k, cos, sin):
    B, H_kv, T, D = k.shape
    out = np.empty_like(k)
    for b in range(B):
        for h in range(H_kv):
            out[b, h] = rope_rotate(k[b, h], cos, sin, np.arange(T))
    return out


@pytest.mark.parametrize("H,H_kv", [(2, 2), (4, 2), (6, 1)])
def test_decode_is_the_last_row_of_the_forward(H, H_kv):
    rng = np.random.default_rng(7)
    B, T, D = 2, 13, 8
    cos, sin = rope_angles_f64(T, D)
    q, k, v = _sequence(rng, B, H, H_kv, T, D)
    scale = 0.3
    o_full, lse_full = attention_forward(q, k, v, cos, sin, None, scale)
    kc = _rotated_cache(k, cos, sin)
    # cache filled to the whole sequence for row 0, to 9 tokens for row 1
    lens = np.array([T, 9])
    o, lse = decode_forward(q[np.arange(B), :, lens - 1], kc, v, lens, cos, sin, scale)
    for b in range(B):
        L = lens[b]
        ob, lseb = attention_forward(q[b:b + 1, :, :L], k[b:b + 1, :, :L], v[b:b + 1, :, :L],
                                     cos, sin, None, scale)
        np.testing.assert_allclose(o[b], ob[0, :, L - 1], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[b], lseb[0, :, L - 1], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(o[0], o_full[0, :, T - 1], rtol=1e-12, atol=1e-12)


def test_decode_single_cached_token_closed_form():
    rng = np.random.default_rng(8)
    q = rng.standard_normal((1, 3, 4))
    kc = rng.standard_normal((1, 3, 5, 4))
    vc = rng.standard_normal((1, 3, 5, 4))
    o, lse = decode_forward(q, kc, vc, np.array([1]), None, None, 0.5)
    np.testing.assert_allclose(o[0], vc[0, :, 0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0], 0.5 * np.einsum("hd,hd->h", q[0], kc[0, :, 0]), rtol=1e-14)


def test_decode_invariants():
    rng = np.random.default_rng(9)
    B, H, T, D = 1, 2, 11, 8
    q = rng.standard_normal((B, H, D))
    kc = rng.standard_normal((B, H, T, D))
    vc = rng.standard_normal((B, H, T, D))
    lens = np.array([7])
    o, lse = decode_forward(q, kc, vc, lens, None, None, 0.25)
    # cached rows past the length are never read
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[:, :, 7:] = 1e6
    vc2[:, :, 7:] = np.nan
    o2, lse2 = decode_forward(q, kc2, vc2, lens, None, None, 0.25)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)
    # all cached tokens are visible: permuting them (keys with values) changes nothing
    perm = rng.permutation(7)
    kc3, vc3 = kc.copy(), vc.copy()
    kc3[:, :, :7] = kc[:, :, perm]
    vc3[:, :, :7] = vc[:, :, perm]
    o3, lse3 = decode_forward(q, kc3, vc3, lens, None, None, 0.25)
    np.testing.assert_allclose(o3, o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse3, lse, rtol=1e-13)
    # o is a convex combination of the visible values
    assert np.all(o <= vc[:, :, :7].max(axis=2) + 1e-12)
    assert np.all(o >= vc[:, :, :7].min(axis=2) - 1e-12)


def test_decode_grouped_heads_equal_repeated_cache():
    rng = np.random.default_rng(10)
    B, H, H_kv, T, D = 2, 6, 2, 9, 4
    cos, sin = rope_angles_f64(T, D)
    q = rng.standard_normal((B, H, D))
    kc = rng.standard_normal((B, H_kv, T, D))
    vc = rng.standard_normal((B, H_kv, T, D))
    lens = np.array([9, 4])
    o, lse = decode_forward(q, kc, vc, lens, cos, sin, 0.5)
    G = H // H_kv
    o2, lse2 = decode_forward(q, np.repeat(kc, G, axis=1), np.repeat(vc, G, axis=1), lens,
                              cos, sin, 0.5)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)
    with pytest.raises(ValueError):
        decode_forward(q, kc[:, :1].repeat(4, axis=1), vc[:, :1].repeat(4, axis=1), lens, cos,
                       sin, 0.5)
    with pytest.raises(ValueError):
        decode_forward(q, kc, vc, np.array([0, 4]), cos, sin, 0.5)


def test_planted_wrong_query_position_is_caught(monkeypatch):
    """A decode oracle that rotates the query at position cache_len (one too
    far) must disagree with the last row of the forward."""
    import oracle.decode as dec

    real = dec.rope_rotate

    def shifted(x, cos, sin, pos):
        return real(x, cos, sin, np.asarray(pos) + 1)

    rng = np.random.default_rng(11)
    B, H, T, D = 1, 2, 12, 8
    cos, sin = rope_angles_f64(T + 1, D)
    q, k, v = _sequence(rng, B, H, H, T, D)
    kc = _rotated_cache(k, cos, sin)
    lens = np.array([T])
    ob, _ = attention_forward(q, k, v, cos, sin, None, 0.4)
    monkeypatch.setattr(dec, "rope_rotate", shifted)
    o, _ = dec.decode_forward(q[:, :, T - 1], kc, v, lens, cos, sin, 0.4)
    assert not np.allclose(o[0], ob[0, :, T - 1], rtol=1e-6, atol=1e-6)
