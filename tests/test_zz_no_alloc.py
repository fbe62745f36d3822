"""attn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Callers embedded in a runtime that has reserved all device memory for its own
pool, or that may not call cudaMalloc/cudaFree on their hot path, cannot pass a
workspace. This entry point uses the library's fixed device scratch array
instead. Its gradients must agree with attn_bwd's (same inputs, same forward)
and with the float64 oracle, within the parity tolerances, on calls in a row:
each later call reuses the array the one before left behind (a different
problem with a different document layout), so stale contents, above all stale
document ranges, must not leak into it.

This file is collected last, so a run that stops at the first failure has run
every other test before it.
"""

import numpy as np
import pytest

from tests.parity import TOL, compare_arrays, oracle_outputs
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


def _flat(d):
    """[B, H, T, D] -> [B*H, T, D] slices, as the parity helpers compare them."""
    return {k: v.reshape((-1,) + v.shape[2:]) for k, v in d.items()}


def test_noalloc_backward_matches_attn_bwd_and_oracle_on_calls_in_a_row():
    _cuda()
    from bwd_causal_sdpa_b200.runner import AttnRunner

    cases = [
        # packed documents with RoPE (document ranges and Delta both in the array)
        make_workload(config_by_name("packed_docs"), B=2, H=3, T=520, doc_min=16, doc_max=200,
                      seed=41),
        # a smaller problem with another document layout: the array still holds
        # the first call's longer ranges past this call's B*T tokens and at
        # other offsets
        make_workload(config_by_name("packed_docs"), B=1, H=2, T=300, D=64, doc_min=5,
                      doc_max=90, seed=42),
        # one document per row, float32 storage (the 1e-5 bound)
        make_workload(config_by_name("tiny_fp32"), seed=43),
    ]
    for w in cases:
        r = AttnRunner.from_workload(w)
        r.forward()
        r.backward()
        ref = r.results()
        got = _noalloc_grads(r)
        tol = TOL[w.dtype]
        keys = ("dq", "dk", "dv")
        compare_arrays(_flat(got), _flat({k: ref[k] for k in keys}), tol, keys=keys)
        orc = oracle_outputs(w)
        compare_arrays(_flat(got), _flat({k: orc[k] for k in keys}), tol, keys=keys)


def test_noalloc_rejects_problems_beyond_its_scratch():
    import bwd_causal_sdpa_b200 as A

    P = 1 << 20  # never dereferenced: the size check fails on the host first
    # 4*B*H*T bytes of Delta alone exceed the 8 MiB array here
    B, H, T = 1, 64, 65536
    rc = A.attn_bwd_noalloc(P, P, P, P, P, P, None, None, None, B, H, T, 64, 0.125,
                            A.ATTN_BF16, P, P, P, None)
    assert rc == A.ATTN_ESCRATCH
    assert "scratch" in A.error_string(rc)

