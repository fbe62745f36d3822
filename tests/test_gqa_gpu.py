"""GPU parity for grouped-query attention (k, v with fewer heads than q).

Small cases cover both storage types, both head sizes, group sizes 2 to 8,
RoPE, packed documents and ragged tails, compared element by element with the
oracle; one full 8K case is compared on a whole sampled group (the oracle's
dk, dv of a shared head need every query head that reads it). A last test
checks the structure directly: o and lse of a grouped call equal, bit for bit,
those of the plain call on k, v repeated over each group.
"""

import numpy as np
import pytest

from tests.parity import compare, gpu_outputs, oracle_outputs, rel_fro
from workloads import config_by_name, make_workload

pytestmark = pytest.mark.gpu


def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


SMALL = [
    # name, overrides (H_kv divides H); several 128-row tiles and a ragged tail
    ("tiny_fp32", dict(H=4, H_kv=2, T=200)),
    ("tiny_fp32", dict(H=6, H_kv=2, T=333, D=128, rope=True, varlen=True, doc_min=1,
                       doc_max=150, seed=41)),
    ("gpt12m_layer", dict(B=2, H=6, H_kv=3, T=300, seed=42)),
    ("long_context_8k", dict(B=1, H=8, H_kv=1, T=700, seed=43)),
    ("long_context_8k", dict(B=2, H=4, H_kv=2, T=1000, seed=44)),
    ("packed_docs", dict(B=2, H=4, H_kv=1, T=777, doc_min=32, doc_max=300, seed=45)),
    ("packed_docs", dict(B=2, H=4, H_kv=2, T=640, D=64, doc_min=1, doc_max=130, seed=46)),
    ("gpt12m_layer", dict(B=1, H=2, H_kv=1, T=1, seed=47)),
    ("decoder237m_layer", dict(B=1, H=4, H_kv=2, T=129, rope=False, seed=48)),
]


@pytest.mark.parametrize("name,over", SMALL, ids=[f"{n}-{i}" for i, (n, _) in enumerate(SMALL)])
def test_grouped_query_small_cases_match_oracle(name, over):
    _cuda()
    w = make_workload(config_by_name(name), **over)
    errs = compare(w, gpu_outputs(w), oracle_outputs(w))
    print(name, over, errs)


def test_grouped_query_full_8k_sampled_group_matches_oracle():
    _cuda()
    # 16 query heads over 4 key/value heads at the full 8K length; the sampled
    # group is key/value head 2 (query heads 8..11).
    w = make_workload(config_by_name("long_context_8k"), H_kv=4)
    heads = [(0, 8), (0, 9), (0, 10), (0, 11)]
    errs = compare(w, gpu_outputs(w), oracle_outputs(w, heads=heads), heads=heads)
    print(errs)


@pytest.mark.parametrize("name,over,heads", [
    # 16 query heads on one key/value head at T = 4096: each group is split
    # over CTAs whose dk, dv parts are added in fp32 (the whole group compared)
    ("long_context_8k", dict(H=16, H_kv=1, T=4096, seed=61), [(0, h) for h in range(16)]),
    # enough key/value heads x key tiles to fill the GPU: no split (two groups compared)
    ("packed_docs", dict(B=4, H=16, H_kv=8, T=1280, seed=62),
     [(0, 0), (0, 1), (3, 14), (3, 15)]),
], ids=["split_groups", "whole_groups"])
def test_grouped_query_group_split_and_whole(name, over, heads):
    _cuda()
    w = make_workload(config_by_name(name), **over)
    errs = compare(w, gpu_outputs(w), oracle_outputs(w, heads=heads), heads=heads)
    print(name, over, errs)


@pytest.mark.parametrize("name,over", [
    ("packed_docs", dict(B=2, H=4, H_kv=2, T=1000, seed=51)),
    ("tiny_fp32", dict(H=4, H_kv=1, T=260, seed=52)),
])
def test_grouped_query_equals_repeated_heads(name, over):
    _cuda()
    w = make_workload(config_by_name(name), **over)
    got = gpu_outputs(w)
    G = w.H // w.kv_heads
    w.k = np.repeat(w.k, G, axis=1)
    w.v = np.repeat(w.v, G, axis=1)
    w.H_kv = None
    rep = gpu_outputs(w)
    # the forward of a query head reads the same key/value data either way
    assert np.array_equal(got["o"], rep["o"])
    assert np.array_equal(got["lse"], rep["lse"])
    # dq and the group sums of dk, dv agree up to accumulation order
    tol = 2e-3 if w.dtype == "bf16" else 1e-5
    assert rel_fro(got["dq"], rep["dq"]) < tol
    # (each repeated head's dk, dv is rounded to the storage type before the
    # sum, so bf16 agrees only to a few storage roundings)
    sum_tol = 1e-2 if w.dtype == "bf16" else 1e-5
    B, _, T, D = rep["dk"].shape
    for key in ("dk", "dv"):
        summed = rep[key].reshape(B, w.H // G, G, T, D).sum(axis=2)
        assert rel_fro(got[key], summed) < sum_tol, key
