"""Both routes of the backward's dQ against the float64 oracle.

The backward forms dQ either beside dK and dV in the key-tile kernel (fp32
reduce-adds into an accumulator, finished by a separate pass) or in its own
query-tile pass (no accumulator); the product library takes one route per
head size, chosen by measurement, and the test build (libattn_debug.so: the
same sources) takes the other. The cases below run through the test build,
so that together with the other parity tests both routes are checked on
every case kind: RoPE with fp16 operands and without, packed documents,
ragged tails, both head sizes and grouped heads (split and whole groups).
"""

import ctypes
import os

import numpy as np
import pytest

from tests.parity import compare, oracle_outputs
from workloads import config_by_name, make_workload

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TEST_LIB = os.path.join(ROOT, "bwd_causal_sdpa_b200", "libattn_debug.so")


def _test_lib():
    import bwd_causal_sdpa_b200 as A

    if not os.path.exists(TEST_LIB):
        pytest.fail(f"{TEST_LIB} is missing: python bwd_causal_sdpa_b200/build.py --debug")
    lib = ctypes.CDLL(TEST_LIB)
    for name, (res, args) in A._SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


CASES = [
    ("long_context_8k", dict(B=1, H=2, T=700, seed=71)),
    ("decoder237m_layer", dict(B=1, H=2, T=515, seed=72)),
    ("packed_docs", dict(B=2, H=2, T=777, doc_min=32, doc_max=300, seed=73)),
    ("packed_docs", dict(B=2, H=2, T=640, D=64, doc_min=1, doc_max=130, seed=74)),
    ("gpt12m_layer", dict(B=1, H=2, T=256, rope=False, seed=75)),
    ("long_context_8k", dict(B=1, H=16, H_kv=1, T=1024, seed=76)),
    ("gpt12m_layer", dict(B=1, H=1, T=1, seed=77)),
]


@pytest.mark.parametrize("name,over", CASES, ids=[f"{n}-{i}" for i, (n, _) in enumerate(CASES)])
def test_other_dq_route_matches_oracle(name, over):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import bwd_causal_sdpa_b200 as A
    from bwd_causal_sdpa_b200.runner import AttnRunner

    lib = _test_lib()
    w = make_workload(config_by_name(name), **over)
    r = AttnRunner.from_workload(w)
    p = r.p
    ptr = lambda t: None if t is None else t.data_ptr()
    ws_bytes = max(lib.attn_workspace_bytes_gqa(p.B, p.H, p.H_kv, p.T, p.D, p.dtype, 0),
                   lib.attn_workspace_bytes_gqa(p.B, p.H, p.H_kv, p.T, p.D, p.dtype, 1))
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=r.device)
    rc = lib.attn_fwd_gqa(ptr(r.q), ptr(r.k), ptr(r.v), ptr(r.rope_cos), ptr(r.rope_sin),
                          ptr(r.cu), ptr(r.o), ptr(r.lse), p.B, p.H, p.H_kv, p.T, p.D, p.scale,
                          p.dtype, ptr(ws), ws_bytes, None)
    assert rc == A.ATTN_OK
    rc = lib.attn_bwd_gqa(ptr(r.q), ptr(r.k), ptr(r.v), ptr(r.o), ptr(r.do), ptr(r.lse),
                          ptr(r.rope_cos), ptr(r.rope_sin), ptr(r.cu), p.B, p.H, p.H_kv, p.T,
                          p.D, p.scale, p.dtype, ptr(r.dq), ptr(r.dk), ptr(r.dv), ptr(ws),
                          ws_bytes, None)
    assert rc == A.ATTN_OK
    assert lib.attn_get_status(None) == A.ATTN_OK
    errs = compare(w, r.results(), oracle_outputs(w))
    print(name, over, errs)
