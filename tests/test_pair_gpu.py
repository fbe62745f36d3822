"""GPU parity for the CTA-pair backward route (attn_set_backward_route(2)).

dK and dV come from the key-tile kernel run on clusters of two CTAs (tcgen05
products of M = 256 keys, one instruction stream for both SMs), dQ from the
query-tile pass. Cases cover an odd number of key tiles (the last pair's
second CTA holds no key), packed documents, a split group of query heads,
bf16 operands (no RoPE), a one-token sequence and the full 8K length on a
sampled head; a D = 64 case checks that it takes the single-CTA route. The
route is reset to the default after each case.
"""

import pytest

from tests.parity import compare, gpu_outputs, oracle_outputs
from workloads import config_by_name, make_workload

pytestmark = pytest.mark.gpu

CASES = [
    ("long_context_8k", dict(B=1, H=2, T=700, seed=81), None),
    ("long_context_8k", dict(B=1, H=2, T=640, seed=82), None),  # 5 key tiles
    ("packed_docs", dict(B=2, H=2, T=777, doc_min=1, doc_max=300, seed=83), None),
    ("long_context_8k", dict(B=1, H=16, H_kv=1, T=1024, seed=84), None),  # group split over CTAs
    ("gpt12m_layer", dict(B=1, H=2, T=300, D=128, rope=False, seed=85), None),
    ("gpt12m_layer", dict(B=1, H=1, T=1, D=128, seed=86), None),
    ("decoder237m_layer", dict(B=1, H=2, T=515, seed=87), None),  # D = 64: single-CTA route
    ("long_context_8k", dict(seed=88), [(0, 5)]),
]


@pytest.mark.parametrize("name,over,heads", CASES, ids=[f"{n}-{i}" for i, (n, _, _) in enumerate(CASES)])
def test_pair_route_matches_oracle(name, over, heads):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import bwd_causal_sdpa_b200 as A

    w = make_workload(config_by_name(name), **over)
    assert A.attn_set_backward_route(2) == A.ATTN_OK
    try:
        got = gpu_outputs(w)
    finally:
        A.attn_set_backward_route(0)
    errs = compare(w, got, oracle_outputs(w, heads=heads), heads=heads)
    print(name, over, errs)

