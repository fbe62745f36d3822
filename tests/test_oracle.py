"""Pins for the float64 oracle (CPU only).

Each test checks the oracle against something other than itself: hand-derived
closed forms (tests/golden), central finite differences of L = sum(o * dO),
invariants that hold for any input, and PyTorch's float64
scaled_dot_product_attention with autograd on the cases it covers. The last
group plants plausible mistakes into a copy of the oracle and checks that at
least one pin catches each.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.attention as A
from oracle import (attention_backward, attention_forward, doc_layout,
                    rope_angles_f64, rope_rotate, rope_rotate_inverse)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")
MATH_NS = {"e": math.e, "cos1": math.cos(1.0), "sin1": math.sin(1.0),
           "log": math.log, "exp": math.exp, "cos": math.cos, "sin": math.sin}


def _ev(expr):
    return float(eval(expr, {"__builtins__": {}}, MATH_NS))  # closed forms from the fixture


def _ev_array(rows):
    return np.asarray([[_ev(x) for x in row] for row in rows], dtype=np.float64)


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _loss(q, k, v, do, cos, sin, cu, scale):
    o, _ = attention_forward(q, k, v, cos, sin, cu, scale)
    return float((o * do).sum())


def _fd_grads(q, k, v, do, cos, sin, cu, scale, eps=1e-6):
    grads = []
    for which in range(3):
        args = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(args[which])
        it = np.nditer(args[which], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            orig = args[which][idx]
            args[which][idx] = orig + eps
            lp = _loss(*args, do, cos, sin, cu, scale)
            args[which][idx] = orig - eps
            lm = _loss(*args, do, cos, sin, cu, scale)
            args[which][idx] = orig
            g[idx] = (lp - lm) / (2 * eps)
        grads.append(g)
    return grads


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


# --------------------------------------------------------------------------
# Worked examples (closed forms derived by hand)
# --------------------------------------------------------------------------

def _golden():
    with open(GOLDEN) as f:
        return {e["name"]: e for e in json.load(f)["examples"]}


@pytest.mark.parametrize("name", ["two_tokens_no_rope", "two_tokens_rope_relative_angle"])
def test_worked_examples(name):
    ex = _golden()[name]
    T, D = ex["T"], ex["D"]
    q = np.asarray(ex["q"], float)[None, None]
    k = np.asarray(ex["k"], float)[None, None]
    v = np.asarray(ex["v"], float)[None, None]
    do = np.asarray(ex["dO"], float)[None, None]
    cos = sin = None
    if ex["rope"]:
        cos, sin = rope_angles_f64(T, D, ex["theta"])
    o, lse = attention_forward(q, k, v, cos, sin, None, ex["scale"])
    exp_o = _ev_array(ex["expected"]["o"])
    exp_lse = np.asarray([_ev(s) for s in ex["expected"]["lse"]])
    np.testing.assert_allclose(o[0, 0], exp_o, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], exp_lse, rtol=1e-14, atol=1e-15)
    if "dq" in ex["expected"]:
        dq, dk, dv = attention_backward(q, k, v, do, cos, sin, None, ex["scale"])
        for got, key in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
            want = _ev_array(ex["expected"][key])
            np.testing.assert_allclose(got[0, 0], want, rtol=1e-14, atol=1e-15)


def test_rope_pairs_are_interleaved():
    ex = _golden()["rope_pairs_are_interleaved"]
    D, pos = ex["D"], ex["pos"]
    cos, sin = rope_angles_f64(pos + 1, D, ex["theta"])
    y = A.rope_rotate(np.asarray([ex["x"]], float), cos, sin, np.asarray([pos]))
    np.testing.assert_allclose(y[0], [_ev(s) for s in ex["expected_rotated"]], rtol=1e-14, atol=1e-16)


# --------------------------------------------------------------------------
# Closed forms
# --------------------------------------------------------------------------

def test_single_token_returns_v_and_zero_lse_offset():
    rng = np.random.default_rng(0)
    q, k, v = (_rand(rng, 2, 3, 1, 8) for _ in range(3))
    o, lse = attention_forward(q, k, v, None, None, None, 0.3)
    np.testing.assert_allclose(o, v, rtol=0, atol=0)
    np.testing.assert_allclose(lse, 0.3 * (q * k).sum(-1), rtol=1e-15)


def test_zero_queries_give_running_mean_and_log_count():
    rng = np.random.default_rng(1)
    T, D = 12, 4
    q = np.zeros((1, 1, T, D))
    k, v = _rand(rng, 1, 1, T, D), _rand(rng, 1, 1, T, D)
    o, lse = attention_forward(q, k, v, None, None, None, 0.5)
    mean = np.cumsum(v[0, 0], axis=0) / np.arange(1, T + 1)[:, None]
    np.testing.assert_allclose(o[0, 0], mean, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], np.log(np.arange(1, T + 1)), rtol=1e-14)


def test_zero_queries_packed_use_document_counts():
    rng = np.random.default_rng(2)
    B, T, D = 2, 10, 4
    cu = np.asarray([0, 3, 10, 14, 20], dtype=np.int32)
    q = np.zeros((B, 1, T, D))
    k, v = _rand(rng, B, 1, T, D), _rand(rng, B, 1, T, D)
    _, lse = attention_forward(q, k, v, None, None, cu, 1.0)
    counts = np.concatenate([np.arange(1, 4), np.arange(1, 8), np.arange(1, 5), np.arange(1, 7)])
    np.testing.assert_allclose(lse.reshape(-1), np.log(counts), rtol=1e-14)


# --------------------------------------------------------------------------
# Library routine: PyTorch float64 SDPA with autograd (no RoPE, one document)
# --------------------------------------------------------------------------

def test_matches_torch_sdpa_float64():
    rng = np.random.default_rng(3)
    B, H, T, D = 2, 3, 17, 8
    q, k, v, do = (_rand(rng, B, H, T, D) for _ in range(4))
    scale = 0.37
    o, lse = attention_forward(q, k, v, None, None, None, scale)
    dq, dk, dv = attention_backward(q, k, v, do, None, None, None, scale)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=scale)
    to.backward(torch.tensor(do))
    np.testing.assert_allclose(o, to.detach().numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-11, atol=1e-12)
    # lse against torch.logsumexp over the explicitly masked scores
    s = torch.tensor(q) @ torch.tensor(k).transpose(-1, -2) * scale
    s = s.masked_fill(~torch.ones(T, T, dtype=torch.bool).tril(), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=1e-13)


# --------------------------------------------------------------------------
# Finite differences (with and without RoPE, with and without packing)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("rope,packed", [(False, False), (True, False), (False, True), (True, True)])
def test_gradients_match_central_differences(rope, packed):
    rng = np.random.default_rng(10 + 2 * rope + packed)
    B, H, T, D = (2, 1, 7, 4) if packed else (1, 2, 6, 4)
    q, k, v, do = (_rand(rng, B, H, T, D) for _ in range(4))
    cu = np.asarray([0, 3, 7, 8, 14], dtype=np.int32) if packed else None
    cos = sin = None
    if rope:
        cos, sin = rope_angles_f64(T, D, 100.0)
    scale = 0.6
    dq, dk, dv = attention_backward(q, k, v, do, cos, sin, cu, scale)
    fq, fk, fv = _fd_grads(q, k, v, do, cos, sin, cu, scale)
    assert _rel(dq, fq) < 1e-7
    assert _rel(dk, fk) < 1e-7
    assert _rel(dv, fv) < 1e-7


# --------------------------------------------------------------------------
# Invariants
# --------------------------------------------------------------------------

def test_softmax_rows_sum_to_one_and_masked_entries_are_zero():
    rng = np.random.default_rng(4)
    T, D = 16, 8
    q, k, v = (_rand(rng, T, D) for _ in range(3))
    pos, start = doc_layout(1, T, np.asarray([0, 5, 16], dtype=np.int32))
    cos, sin = rope_angles_f64(T, D)
    f = A.forward_head(q * 3, k * 3, v, cos, sin, pos[0], start[0], 0.5)
    P = f["P"]
    assert np.max(np.abs(P.sum(axis=1) - 1.0)) < 1e-12
    assert np.all(P[~f["allowed"]] == 0.0)
    assert np.all(P[f["allowed"]] > 0.0)


def test_causality_future_tokens_do_not_change_earlier_outputs():
    rng = np.random.default_rng(5)
    B, H, T, D = 1, 2, 12, 8
    q, k, v = (_rand(rng, B, H, T, D) for _ in range(3))
    cos, sin = rope_angles_f64(T, D)
    o1, l1 = attention_forward(q, k, v, cos, sin, None, 0.4)
    for i in range(T - 1):
        k2, v2, q2 = k.copy(), v.copy(), q.copy()
        k2[:, :, i + 1:] += _rand(rng, B, H, T - i - 1, D)
        v2[:, :, i + 1:] += _rand(rng, B, H, T - i - 1, D)
        q2[:, :, i + 1:] += _rand(rng, B, H, T - i - 1, D)
        o2, l2 = attention_forward(q2, k2, v2, cos, sin, None, 0.4)
        assert np.array_equal(o1[:, :, : i + 1], o2[:, :, : i + 1])
        assert np.array_equal(l1[:, :, : i + 1], l2[:, :, : i + 1])


def test_rope_preserves_norms_and_identity_at_position_zero():
    rng = np.random.default_rng(6)
    T, D = 50, 16
    cos, sin = rope_angles_f64(T, D)
    x = _rand(rng, T, D)
    pos = np.arange(T)
    y = rope_rotate(x, cos, sin, pos)
    assert np.max(np.abs(np.linalg.norm(y, axis=1) - np.linalg.norm(x, axis=1))) < 1e-13
    # pairwise norms too (each pair is rotated on its own)
    pn = lambda a: a[:, 0::2] ** 2 + a[:, 1::2] ** 2
    assert np.max(np.abs(pn(y) - pn(x))) < 1e-12
    z = rope_rotate(x, cos, sin, np.zeros(T, dtype=np.int64))
    assert np.array_equal(z, x)
    # the inverse undoes the rotation
    assert np.max(np.abs(rope_rotate_inverse(y, cos, sin, pos) - x)) < 1e-13


def test_rope_scores_depend_only_on_relative_position():
    rng = np.random.default_rng(7)
    D = 16
    cos, sin = rope_angles_f64(200, D)
    q, k = _rand(rng, 1, D), _rand(rng, 1, D)
    for m, n, shift in [(5, 2, 40), (17, 17, 3), (3, 30, 100), (0, 9, 77)]:
        a = rope_rotate(q, cos, sin, np.asarray([m])) @ rope_rotate(k, cos, sin, np.asarray([n])).T
        b = rope_rotate(q, cos, sin, np.asarray([m + shift])) @ rope_rotate(k, cos, sin, np.asarray([n + shift])).T
        assert abs(a - b).max() < 1e-12


def test_packed_documents_equal_separate_runs():
    rng = np.random.default_rng(8)
    B, H, T, D = 2, 2, 20, 8
    cu = np.asarray([0, 6, 7, 20, 31, 40], dtype=np.int32)
    q, k, v, do = (_rand(rng, B, H, T, D) for _ in range(4))
    cos, sin = rope_angles_f64(T, D)
    o, lse = attention_forward(q, k, v, cos, sin, cu, 0.35)
    dq, dk, dv = attention_backward(q, k, v, do, cos, sin, cu, 0.35)
    for a, e in zip(cu[:-1], cu[1:]):
        b, lo, hi = a // T, a % T, e - (a // T) * T
        sl = lambda x: x[b:b + 1, :, lo:hi].copy()
        o1, l1 = attention_forward(sl(q), sl(k), sl(v), cos, sin, None, 0.35)
        g = attention_backward(sl(q), sl(k), sl(v), sl(do), cos, sin, None, 0.35)
        np.testing.assert_allclose(o[b:b + 1, :, lo:hi], o1, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse[b:b + 1, :, lo:hi], l1, rtol=1e-13, atol=1e-14)
        for got, want in zip((dq, dk, dv), g):
            np.testing.assert_allclose(got[b:b + 1, :, lo:hi], want, rtol=1e-12, atol=1e-13)


def test_gradient_identities():
    rng = np.random.default_rng(9)
    T, D = 14, 8
    q, k, v, do = (_rand(rng, T, D) for _ in range(4))
    pos, start = doc_layout(1, T, None)
    g = A.backward_head(q, k, v, do, None, None, pos[0], start[0], 0.5)
    assert np.max(np.abs(g["dS"].sum(axis=1))) < 1e-12          # sum_j dS_ij = 0
    np.testing.assert_allclose(g["dv"].sum(axis=0), do.sum(axis=0), rtol=1e-12, atol=1e-12)
    assert np.max(np.abs(g["dk"].sum(axis=0))) < 1e-12          # sum_j dk_j = 0 without RoPE


def test_grouped_query_attention_gradients_match_central_differences():
    rng = np.random.default_rng(30)
    B, H, H_kv, T, D = 1, 4, 2, 6, 4
    q, do = _rand(rng, B, H, T, D), _rand(rng, B, H, T, D)
    k, v = _rand(rng, B, H_kv, T, D), _rand(rng, B, H_kv, T, D)
    cos, sin = rope_angles_f64(T, D, 100.0)
    dq, dk, dv = attention_backward(q, k, v, do, cos, sin, None, 0.6)
    fq, fk, fv = _fd_grads(q, k, v, do, cos, sin, None, 0.6)
    assert _rel(dq, fq) < 1e-7
    assert _rel(dk, fk) < 1e-7
    assert _rel(dv, fv) < 1e-7


def test_grouped_query_attention_equals_repeated_heads():
    # GQA is MHA on key/value heads repeated over each group; the shared
    # heads' gradients are the sums over their group (chain rule).
    rng = np.random.default_rng(31)
    B, H, H_kv, T, D = 2, 6, 2, 9, 8
    q, do = _rand(rng, B, H, T, D), _rand(rng, B, H, T, D)
    k, v = _rand(rng, B, H_kv, T, D), _rand(rng, B, H_kv, T, D)
    cu = np.asarray([0, 4, 9, 12, 18], dtype=np.int32)
    cos, sin = rope_angles_f64(T, D)
    kr, vr = np.repeat(k, H // H_kv, axis=1), np.repeat(v, H // H_kv, axis=1)
    o, lse = attention_forward(q, k, v, cos, sin, cu, 0.4)
    o2, lse2 = attention_forward(q, kr, vr, cos, sin, cu, 0.4)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)
    dq, dk, dv = attention_backward(q, k, v, do, cos, sin, cu, 0.4)
    dq2, dk2, dv2 = attention_backward(q, kr, vr, do, cos, sin, cu, 0.4)
    np.testing.assert_allclose(dq, dq2, rtol=1e-13, atol=1e-14)
    g = H // H_kv
    np.testing.assert_allclose(dk, dk2.reshape(B, H_kv, g, T, D).sum(axis=2), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(B, H_kv, g, T, D).sum(axis=2), rtol=1e-12, atol=1e-13)
    with pytest.raises(ValueError):
        attention_forward(q, k[:, :1].repeat(4, axis=1), v[:, :1].repeat(4, axis=1), None, None, None, 1.0)


def test_doc_layout_rejects_bad_boundaries():
    with pytest.raises(ValueError):
        doc_layout(2, 8, np.asarray([0, 5, 12, 16], dtype=np.int32))   # doc crosses row 0 -> 1
    with pytest.raises(ValueError):
        doc_layout(1, 8, np.asarray([0, 5, 5, 8], dtype=np.int32))     # not strictly rising
    with pytest.raises(ValueError):
        doc_layout(1, 8, np.asarray([0, 5, 7], dtype=np.int32))        # does not end at B*T


# --------------------------------------------------------------------------
# Planted mistakes: every mutant must fail at least one pin
# --------------------------------------------------------------------------

def _pins_pass():
    """A compact run of the pins above; returns False when any fails."""
    checks = [test_gradients_match_central_differences,
              test_matches_torch_sdpa_float64,
              test_zero_queries_give_running_mean_and_log_count,
              test_rope_pairs_are_interleaved,
              lambda: test_worked_examples("two_tokens_no_rope"),
              lambda: test_worked_examples("two_tokens_rope_relative_angle")]
    for c in checks:
        try:
            if c is test_gradients_match_central_differences:
                c(True, True)
            else:
                c()
        except (AssertionError, ValueError):
            return False
    return True


_orig_rotate = A.rope_rotate
_orig_inverse = A.rope_rotate_inverse
_orig_allowed = A.allowed_keys
_orig_softmax = A._softmax_three_pass
_orig_backward = A.backward_head


def _mut_half_split(x, cos, sin, pos):
    c, s = cos[pos], sin[pos]
    h = x.shape[1] // 2
    y = np.empty_like(x)
    y[:, :h] = x[:, :h] * c - x[:, h:] * s
    y[:, h:] = x[:, :h] * s + x[:, h:] * c
    return y


def _mut_strict_causal(doc_start):
    m = _orig_allowed(doc_start)
    T = m.shape[0]
    m = m & ~np.eye(T, dtype=bool)
    m[0, 0] = True
    return m


def _mut_lse_no_log(S, allowed):
    Sm = np.where(allowed, S, -np.inf)
    m = Sm.max(axis=1, keepdims=True)
    e = np.exp(Sm - m)
    l = e.sum(axis=1, keepdims=True)
    return e / l, (m + l)[:, 0]


def _mut_no_delta(q, k, v, do, cos, sin, pos, doc_start, scale, fwd=None):
    f = A.forward_head(q, k, v, cos, sin, pos, doc_start, scale)
    P = f["P"]
    dS = P * (do @ v.T)
    dv = P.T @ do
    dqr, dkr = scale * (dS @ f["kr"]), scale * (dS.T @ f["qr"])
    if cos is not None:
        return {"dq": _orig_inverse(dqr, cos, sin, pos), "dk": _orig_inverse(dkr, cos, sin, pos), "dv": dv, "dS": dS}
    return {"dq": dqr, "dk": dkr, "dv": dv, "dS": dS}


def _mut_dk_transposed_operand(q, k, v, do, cos, sin, pos, doc_start, scale, fwd=None):
    g = _orig_backward(q, k, v, do, cos, sin, pos, doc_start, scale, fwd)
    f = g["fwd"]
    dkr = scale * (g["dS"] @ f["qr"])      # dS instead of dS^T
    g["dk"] = _orig_inverse(dkr, cos, sin, pos) if cos is not None else dkr
    return g


MUTANTS = {
    "inverse_rope_uses_forward_rotation": ("rope_rotate_inverse", lambda g, c, s, p: _orig_rotate(g, c, s, p)),
    "rope_half_split_pairs": ("rope_rotate", _mut_half_split),
    "diagonal_masked": ("allowed_keys", _mut_strict_causal),
    "lse_missing_log": ("_softmax_three_pass", _mut_lse_no_log),
    "dS_without_delta": ("backward_head", _mut_no_delta),
    "dk_uses_dS_not_transposed": ("backward_head", _mut_dk_transposed_operand),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_is_caught(mutant, monkeypatch):
    assert _pins_pass()
    attr, fn = MUTANTS[mutant]
    monkeypatch.setattr(A, attr, fn)
    assert not _pins_pass(), f"no pin caught the planted mistake {mutant}"
