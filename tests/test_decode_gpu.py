"""GPU parity for decode attention (one new token against a key/value cache)
through the C ABI, against the float64 decode oracle: small cases element by
element (both storage types and head sizes, group sizes 1 to 32, cache
lengths 1, ragged, a multiple of the 128-token chunk and the full capacity),
the two named decode workloads on sampled heads, cache rows past the length
(set to NaN) without effect on the result, and out-of-range lengths reported
and clamped. With up to 148 cached heads the persistent streaming kernel
splits the cached tokens of all heads into one equal span per CTA, so the
small cases put each head over several CTAs (partials merged by the head's
last CTA) and decode_8k_gqa mixes heads held whole with split ones; with
more cached heads (decode_237m, and two small cases) the split tensor-core
kernel and its combine run."""

import numpy as np
import pytest

from oracle import decode_forward
from tests.parity import rel_fro
from workloads import decode_config_by_name, make_decode_workload

pytestmark = pytest.mark.gpu

TOL = {"bf16": {"o": 1e-2, "lse": 1e-4}, "f32": {"o": 1e-5, "lse": 1e-5}}


def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _run(w):
    from bwd_causal_sdpa_b200 import ATTN_OK
    from bwd_causal_sdpa_b200.runner import DecodeRunner

    r = DecodeRunner(w)
    r.run()
    assert r.status() == ATTN_OK
    return r.results()


def _compare(w, got, heads=None):
    o, lse = decode_forward(w.q, w.k_cache, w.v_cache, w.cache_lens, w.rope_cos, w.rope_sin,
                            w.scale, heads=heads)
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    idx = tuple(np.array(heads).T)
    errs = {"o": rel_fro(got["o"][idx], o[idx]), "lse": rel_fro(got["lse"][idx], lse[idx])}
    tol = TOL[w.dtype]
    assert np.all(np.isfinite(got["o"][idx])) and np.all(np.isfinite(got["lse"][idx]))
    assert errs["o"] <= tol["o"] and errs["lse"] <= tol["lse"], errs
    return errs


SMALL = [
    ("decode_237m", dict(B=3, H=4, H_kv=4, T_max=300, len_min=1, seed=31)),
    ("decode_237m", dict(B=2, H=8, H_kv=2, T_max=700, len_min=600, seed=32)),
    ("decode_8k_gqa", dict(B=2, H=8, H_kv=1, T_max=1000, len_min=1, seed=33)),
    ("decode_8k_gqa", dict(B=3, H=6, H_kv=3, T_max=512, len_min=512, seed=34)),
    ("decode_8k_gqa", dict(B=2, H=4, H_kv=4, T_max=257, len_min=1, seed=35, rope=False)),
    ("decode_8k_gqa", dict(B=2, H=16, H_kv=2, T_max=384, len_min=100, seed=36, dtype="f32")),
    ("decode_237m", dict(B=2, H=2, H_kv=1, T_max=200, len_min=1, seed=37, dtype="f32")),
    # 32 query heads per cached head: bf16 beyond the tensor-core variant's 16 rows
    ("decode_8k_gqa", dict(B=2, H=32, H_kv=1, T_max=300, len_min=1, seed=41)),
    # 12 and 16 query heads per cached head: two 8-head column tiles
    ("decode_8k_gqa", dict(B=2, H=24, H_kv=2, T_max=700, len_min=1, seed=42)),
    ("decode_237m", dict(B=3, H=16, H_kv=1, T_max=400, len_min=200, seed=43)),
    # fewer cached tokens than CTAs: most spans are empty, heads split finely
    ("decode_8k_gqa", dict(B=1, H=4, H_kv=1, T_max=64, len_min=1, seed=44)),
    # more cached heads than SMs: the split tensor-core kernel and its combine
    ("decode_237m", dict(B=20, H=16, H_kv=8, T_max=200, len_min=1, seed=45)),
    ("decode_8k_gqa", dict(B=38, H=16, H_kv=4, T_max=300, len_min=1, seed=46)),
]


@pytest.mark.parametrize("name,over", SMALL, ids=[f"{n}-{i}" for i, (n, _) in enumerate(SMALL)])
def test_decode_small_cases_match_oracle(name, over):
    _cuda()
    w = make_decode_workload(decode_config_by_name(name), **over)
    print(name, over, _compare(w, _run(w)))


def test_decode_lengths_one_and_chunk_multiples():
    _cuda()
    w = make_decode_workload(decode_config_by_name("decode_8k_gqa"), B=4, H=8, H_kv=2,
                             T_max=512, seed=38)
    w.cache_lens = np.array([1, 128, 256, 512], dtype=np.int32)
    print(_compare(w, _run(w)))


@pytest.mark.parametrize("name,heads", [
    ("decode_8k_gqa", [(0, 0), (3, 17), (7, 31)]),
    ("decode_237m", [(0, 0), (9, 8), (15, 15)]),
])
def test_decode_full_size_sampled_heads(name, heads):
    _cuda()
    w = make_decode_workload(decode_config_by_name(name))
    print(name, _compare(w, _run(w), heads=heads))


def test_decode_never_reads_past_the_cache_length():
    _cuda()
    w = make_decode_workload(decode_config_by_name("decode_237m"), B=2, H=4, H_kv=2, T_max=400,
                             len_min=50, seed=39)
    ref = _run(w)
    for b in range(w.B):
        w.k_cache[b, :, w.cache_lens[b]:] = np.nan
        w.v_cache[b, :, w.cache_lens[b]:] = np.nan
    got = _run(w)
    assert np.array_equal(got["o"], ref["o"]) and np.array_equal(got["lse"], ref["lse"])


def test_decode_out_of_range_lengths_are_reported_and_clamped():
    _cuda()
    from bwd_causal_sdpa_b200 import ATTN_EDEVICE_INPUT, ATTN_OK
    from bwd_causal_sdpa_b200.runner import DecodeRunner

    w = make_decode_workload(decode_config_by_name("decode_237m"), B=2, H=2, H_kv=2, T_max=300,
                             seed=40)
    w.cache_lens = np.array([0, 301], dtype=np.int32)
    r = DecodeRunner(w)
    r.run()
    assert r.status() == ATTN_EDEVICE_INPUT
    assert r.status() == ATTN_OK
    got = r.results()
    w.cache_lens = np.array([1, 300], dtype=np.int32)
    _compare(w, got)
