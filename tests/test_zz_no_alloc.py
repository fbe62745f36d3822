"""attn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Callers embedded in a runtime that has reserved all device memory for its own
pool, or that may not call cudaMalloc/cudaFree on their hot path, cannot pass a
workspace. This entry point uses the library's fixed device scratch array
instead. Its gradients must agree with attn_bwd's (same inputs, same forward)
within the parity tolerances, on two calls in a row: the second call reuses
the array the first one left behind, so stale contents must not leak into it.

This file is collected last, so a run that stops at the first failure has run
every other test before it.
"""

import numpy as np
import pytest

from tests.parity import TOL, rel_fro
from workloads import config_by_name, make_workload

pytestmark = pytest.mark.gpu


def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _noalloc_grads(r):
    import torch

    import bwd_causal_sdpa_b200 as A

    p = r.p
    dq, dk, dv = (torch.full_like(r.dq, float("nan")) for _ in range(3))
    rc = A.attn_bwd_noalloc(r.q, r.k, r.v, r.o, r.do, r.lse, r.rope_cos, r.rope_sin, r.cu,
                            p.B, p.H, p.T, p.D, p.scale, p.dtype, dq, dk, dv, r.stream)
    assert rc == A.ATTN_OK, A.error_string(rc)
    assert r.status() == A.ATTN_OK
    f = lambda t: t.to(torch.float64).cpu().numpy()
    return {"dq": f(dq), "dk": f(dk), "dv": f(dv)}


def test_noalloc_backward_matches_attn_bwd_on_two_calls_in_a_row():
    _cuda()
    from bwd_causal_sdpa_b200.runner import AttnRunner

    cases = [
        # packed documents with RoPE (document ranges and Delta both in the array)
        make_workload(config_by_name("packed_docs"), B=2, H=3, T=520, doc_min=16, doc_max=200,
                      seed=41),
        # a different, smaller problem without packing: the array still holds
        # the first call's larger contents
        make_workload(config_by_name("gpt12m_layer"), B=1, H=2, T=300, seed=42),
    ]
    for w in cases:
        r = AttnRunner.from_workload(w)
        r.forward()
        r.backward()
        ref = r.results()
        got = _noalloc_grads(r)
        tol = TOL[w.dtype]
        for key in ("dq", "dk", "dv"):
            assert np.all(np.isfinite(got[key])), key
            err = rel_fro(got[key], ref[key])
            assert err <= tol[key], f"{w.cfg.name} {key}: {err} > {tol[key]}"


def test_noalloc_rejects_problems_beyond_its_scratch():
    import bwd_causal_sdpa_b200 as A

    P = 1 << 20  # never dereferenced: the size check fails on the host first
    # 4*B*H*T bytes of Delta alone exceed the 8 MiB array here
    B, H, T = 1, 64, 65536
    rc = A.attn_bwd_noalloc(P, P, P, P, P, P, None, None, None, B, H, T, 64, 0.125,
                            A.ATTN_BF16, P, P, P, None)
    assert rc == A.ATTN_ESCRATCH
    assert "scratch" in A.error_string(rc)
