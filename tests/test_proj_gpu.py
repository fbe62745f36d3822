"""Parity of the projection GEMMs (QKV projection with its head layout and
RoPE, output projection, and their backward products) with the float64
oracle, element by element over whole tensors.

Tolerances: ||got - ref||_F / ||ref||_F <= 1e-2 for the bf16 outputs (q, k,
v, y, dx, d_o: products of bf16 operands accumulated in fp32 and rounded to
bf16 once, so about 2^-9 relative per element) and <= 1e-3 for the fp32
weight gradients, whose operands are the bf16 inputs themselves (accumulated
in fp32 over B*T terms, never rounded). With RoPE the backward first rotates
dq, dk back and rounds them to bf16 (the tensor-core operand type), so
dw_qkv then carries that one rounding: the bf16 bound applies to it.
"""

import numpy as np
import pytest

from oracle import (attention_forward, out_projection, out_projection_backward, qkv_projection,
                    qkv_projection_backward)
from tests.parity import rel_fro
from workloads import make_proj_workload, proj_config_by_name

pytestmark = pytest.mark.gpu

TOL_BF16 = 1e-2
TOL_F32 = 1e-3


def _run(w, rope):
    from bwd_causal_sdpa_b200 import ATTN_OK
    from bwd_causal_sdpa_b200.runner import ProjRunner

    r = ProjRunner(w, rope=rope)
    r.qkv()
    r.qkv_bwd()
    r.out()
    r.out_bwd()
    assert r.status() == ATTN_OK
    return r, r.results()


def _check(w, got, rope):
    c = w.cfg
    rc, rs = (w.rope_cos, w.rope_sin) if rope else (None, None)
    q, k, v = qkv_projection(w.x, w.w_qkv, c.H, c.H_kv, c.D, rc, rs, w.cu_seqlens)
    dx, dw = qkv_projection_backward(w.dq, w.dk, w.dv, w.x, w.w_qkv, rc, rs, w.cu_seqlens)
    y = out_projection(w.o, w.w_o)
    d_o, dw_o = out_projection_backward(w.dy, w.o, w.w_o)
    errs = {"q": rel_fro(got["q"], q), "k": rel_fro(got["k"], k), "v": rel_fro(got["v"], v),
            "y": rel_fro(got["y"], y), "dx": rel_fro(got["dx"], dx),
            "d_o": rel_fro(got["d_o"], d_o)}
    errs32 = {"dw_qkv": rel_fro(got["dw_qkv"], dw), "dw_o": rel_fro(got["dw_o"], dw_o)}
    for name, arr in got.items():
        assert np.all(np.isfinite(arr)), name
    bad = {k_: e for k_, e in errs.items() if not e <= TOL_BF16}
    tol_dw_qkv = TOL_BF16 if rope else TOL_F32
    bad.update({k_: e for k_, e in errs32.items()
                if not e <= (tol_dw_qkv if k_ == "dw_qkv" else TOL_F32)})
    assert not bad, (c.name, bad, errs, errs32)


@pytest.mark.parametrize("name", ["proj_small_d64", "proj_small_d128"])
@pytest.mark.parametrize("rope", [False, True])
def test_small_projections_match_oracle(name, rope):
    w = make_proj_workload(proj_config_by_name(name))
    _, got = _run(w, rope)
    _check(w, got, rope)


@pytest.mark.parametrize("C,H,H_kv,D,T", [(8, 1, 1, 64, 128), (24, 1, 1, 128, 128),
                                         (1000, 5, 5, 64, 128), (304, 3, 1, 64, 384)])
def test_edge_shapes(C, H, H_kv, D, T):
    # one or three 128-token tiles (256-row pair tiles with an empty or a
    # half-empty second CTA), K below one 64-wide block, with a tail or with an
    # odd number of blocks (a last stage of one block), N tails
    w = make_proj_workload(proj_config_by_name("proj_small_d64"), B=1, T=T, C=C, H=H,
                           H_kv=H_kv, D=D, packed=False, seed=40 + C)
    _, got = _run(w, True)
    _check(w, got, True)


@pytest.mark.parametrize("name", ["proj_237m", "proj_gqa_8k"])
def test_full_size_projections_match_oracle(name):
    w = make_proj_workload(proj_config_by_name(name))
    _, got = _run(w, True)
    _check(w, got, True)


def test_rope_in_projection_feeds_attention_without_rope():
    """x -> attn_qkv_proj (RoPE on) -> attn_fwd_gqa (RoPE off) against the
    oracle's projection followed by its attention."""
    import torch

    from bwd_causal_sdpa_b200 import (ATTN_BF16, attn_fwd_gqa, attn_workspace_bytes_gqa, check)

    w = make_proj_workload(proj_config_by_name("proj_small_d64"))
    c = w.cfg
    r, _ = _run(w, True)
    o = torch.empty_like(r.q)
    lse = torch.empty((c.B, c.H, c.T), dtype=torch.float32, device=r.q.device)
    nb = attn_workspace_bytes_gqa(c.B, c.H, c.H_kv, c.T, c.D, ATTN_BF16, 0)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=r.q.device)
    scale = 1.0 / np.sqrt(c.D)
    check(attn_fwd_gqa(r.q, r.k, r.v, None, None, r.cu, o, lse, c.B, c.H, c.H_kv, c.T, c.D,
                       scale, ATTN_BF16, ws, nb), "attn_fwd_gqa")
    torch.cuda.synchronize()
    q, k, v = qkv_projection(w.x, w.w_qkv, c.H, c.H_kv, c.D, w.rope_cos, w.rope_sin, w.cu_seqlens)
    o_ref, lse_ref = attention_forward(q, k, v, None, None, w.cu_seqlens, scale)
    got_o = o.to(torch.float64).cpu().numpy()
    got_l = lse.to(torch.float64).cpu().numpy()
    assert rel_fro(got_o, o_ref) <= TOL_BF16
    assert rel_fro(got_l, lse_ref) <= 1e-3
