"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Small cases span several 128-row tiles plus a ragged tail and are compared on
every element; the five full-size workloads (in the launch configuration the
benchmark times) are compared on whole sampled (batch, head) slices, which the
oracle computes exactly. Bounds: relative Frobenius error 1e-2 for o, dq, dk,
dv and 1e-4 for lse with bf16 storage; 1e-5 for all five with float32.
"""

import numpy as np
import pytest

from tests.parity import compare, gpu_outputs, oracle_outputs
from workloads import config_by_name, make_workload

pytestmark = pytest.mark.gpu


def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


SMALL = [
    # name, overrides: several tiles and a ragged tail each
    ("tiny_fp32", {}),
    ("tiny_fp32", dict(H=2, T=333, D=128, rope=True, varlen=True, doc_min=1, doc_max=150, seed=11)),
    ("gpt12m_layer", dict(B=2, H=2, T=300)),
    ("decoder237m_layer", dict(B=1, H=2, T=515)),
    ("long_context_8k", dict(B=1, H=2, T=700)),
    ("packed_docs", dict(B=2, H=2, T=777, doc_min=32, doc_max=300)),
    ("packed_docs", dict(B=2, H=1, T=640, D=64, doc_min=1, doc_max=130, seed=12)),
    ("gpt12m_layer", dict(B=1, H=1, T=1, seed=13)),
    ("long_context_8k", dict(B=1, H=1, T=1, seed=14)),
    ("gpt12m_layer", dict(B=1, H=2, T=127, seed=15)),
    ("gpt12m_layer", dict(B=1, H=2, T=129, seed=16)),
    ("long_context_8k", dict(B=2, H=1, T=1000, seed=17)),
    ("gpt12m_layer", dict(B=1, H=2, T=256, rope=False, seed=18)),
]


@pytest.mark.parametrize("name,over", SMALL, ids=[f"{n}-{i}" for i, (n, _) in enumerate(SMALL)])
def test_small_cases_match_oracle(name, over):
    _cuda()
    w = make_workload(config_by_name(name), **over)
    errs = compare(w, gpu_outputs(w), oracle_outputs(w))
    print(name, over, errs)


def _set_cu(w, cu):
    w.cu_seqlens = np.asarray(cu, dtype=np.int32)
    return w


@pytest.mark.parametrize("cu_kind", ["tile_boundaries", "length_one_docs"])
@pytest.mark.parametrize("D", [64, 128])
def test_document_edges(cu_kind, D):
    """Documents on 128-row tile boundaries (every key tile inside one
    document that starts at or before it: the backward's epilogue takes the
    RoPE table rows of such a tile in one block) and documents that cut
    through tiles (per-row table entries), at both head sizes."""
    _cuda()
    T = 384
    w = make_workload(config_by_name("packed_docs"), B=2, H=2, T=T, D=D, varlen=False, seed=21)
    if cu_kind == "tile_boundaries":
        cu = [0, 128, 256, 384, 384 + 1, 384 + 128, 384 + 255, 768]
    else:
        cu = [0, 1, 2, 3, 130, 131, 384, 385, 386, 700, 767, 768]
    _set_cu(w, cu)
    errs = compare(w, gpu_outputs(w), oracle_outputs(w))
    print(cu_kind, D, errs)


FULL = [("tiny_fp32", None), ("gpt12m_layer", [(0, 0), (15, 5)]),
        ("decoder237m_layer", [(0, 0), (7, 15)]), ("long_context_8k", [(0, 9)]),
        ("packed_docs", [(0, 0), (3, 15)])]


@pytest.mark.parametrize("name,heads", FULL, ids=[n for n, _ in FULL])
def test_full_size_sampled_heads_match_oracle(name, heads):
    _cuda()
    w = make_workload(config_by_name(name))
    errs = compare(w, gpu_outputs(w), oracle_outputs(w, heads=heads), heads=heads)
    print(name, errs)


def test_malformed_cu_seqlens_reports_status_and_falls_back():
    _cuda()
    from bwd_causal_sdpa_b200 import ATTN_EDEVICE_INPUT, ATTN_OK
    from bwd_causal_sdpa_b200.runner import AttnRunner

    w = make_workload(config_by_name("gpt12m_layer"), B=2, H=1, T=200, seed=31)
    ref = oracle_outputs(w)  # one document per row
    # B*T + 1 entries, so the device walk stays inside the buffer; the
    # sequence falls at index 2, which makes it malformed.
    bad = np.arange(0, 2 * 200 + 1, dtype=np.int32)
    bad[2] = 0
    w.cu_seqlens = bad
    r = AttnRunner.from_workload(w)
    r.forward()
    r.backward()
    assert r.status() == ATTN_EDEVICE_INPUT
    assert r.status() == ATTN_OK  # cleared by the read
    w.cu_seqlens = None
    compare(w, r.results(), ref)


# ---------------------------------------------------------------------------
# Magnitudes and signs of the score scale. With RoPE the forward stores the
# rotated q and k as fp16 with one power-of-two factor per 128-row tile (each
# tile's largest magnitude brought into [2^14, 2^15)) and folds the factors
# into the score scale; these cases drive tiles far outside fp16's own range
# in both directions, tiles of different magnitudes in one head, and negative
# and zero scales, against the oracle through the C ABI.
# ---------------------------------------------------------------------------

def _scaled(w, q_tiles=(1.0,), k_tiles=(1.0,), scale=None):
    """Multiply q and k by a factor per 128-row tile (cycling through the
    given factors), round back to bf16 and set the score scale."""
    from workloads import round_to_bf16

    def apply(x, facs):
        f = np.array([facs[(t // 128) % len(facs)] for t in range(x.shape[2])], np.float32)
        return round_to_bf16(x * f[None, None, :, None])

    w.q = apply(w.q, q_tiles)
    w.k = apply(w.k, k_tiles)
    if scale is not None:
        w.scale = float(scale)
    return w


MAGNITUDES = [
    # name, q factors per tile, k factors per tile, scale multiplier
    ("large_q_k", (2e4,), (2e4,), 1 / 4e8),        # every tile scaled down, max |x| ~ 1e5 > 65504
    ("tiny_q_k", (1e-5,), (1e-5,), 1e10),         # fp16 subnormal range without the factors
    ("large_q_tiny_k", (3e4,), (3e-5,), 1.0),
    ("mixed_tiles", (1.0, 4.0, 0.5), (1.0, 0.25, 3.0), 1.0),
    ("mixed_extreme", (2e4, 1.0), (1.0, 1e-4), 1 / 2e4),
]


@pytest.mark.parametrize("name,fq,fk,smul", MAGNITUDES, ids=[m[0] for m in MAGNITUDES])
@pytest.mark.parametrize("D", [64, 128])
def test_tile_factor_magnitudes_match_oracle(name, fq, fk, smul, D):
    _cuda()
    w = make_workload(config_by_name("packed_docs"), B=2, H=2, T=600, D=D, doc_min=40,
                      doc_max=400, seed=51)
    w = _scaled(w, fq, fk, w.scale * smul)
    errs = compare(w, gpu_outputs(w), oracle_outputs(w))
    print(name, D, errs)


@pytest.mark.parametrize("sign", ["negative", "zero"])
@pytest.mark.parametrize("rope", [True, False])
def test_negative_and_zero_scale_match_oracle(sign, rope):
    _cuda()
    w = make_workload(config_by_name("packed_docs"), B=2, H=2, T=400, D=128, rope=rope,
                      doc_min=30, doc_max=300, seed=52)
    w = _scaled(w, (1.0, 3.0), (2.0, 0.5), -w.scale if sign == "negative" else 0.0)
    errs = compare(w, gpu_outputs(w), oracle_outputs(w))
    print(sign, rope, errs)


def test_tile_factors_on_grouped_heads_match_oracle():
    _cuda()
    w = make_workload(config_by_name("long_context_8k"), B=1, H=4, H_kv=2, T=520, seed=53)
    w = _scaled(w, (5e3, 1.0, 0.01), (1.0, 7e-3), w.scale / 5e3)
    errs = compare(w, gpu_outputs(w), oracle_outputs(w))
    print(errs)
