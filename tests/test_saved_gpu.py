"""GPU parity for the saved-operand pair attn_fwd_save / attn_bwd_saved.

The backward reads the rotated fp16 q, k and their tile factors that the
forward left in the caller's buffer instead of rotating q, k again. Each case
is compared element by element with the oracle, and with the plain
attn_fwd / attn_bwd pair on the same inputs. The kernels see the same values
either way, so o and lse must be identical bit for bit; dq (and dk, dv when a
key/value group is split over CTAs) are sums that CTAs add into fp32
accumulators in whatever order they finish, so those may differ by the
rounding of that order: at most one bf16 rounding step per element.
"""

import numpy as np
import pytest

from tests.parity import compare, oracle_outputs
from workloads import config_by_name, make_workload

pytestmark = pytest.mark.gpu

CASES = [
    ("long_context_8k", dict(B=1, H=4, T=700, seed=71)),
    ("packed_docs", dict(B=2, H=4, T=777, doc_min=1, doc_max=300, seed=72)),
    ("packed_docs", dict(B=2, H=4, H_kv=2, T=640, D=64, doc_min=16, doc_max=200, seed=73)),
    ("decoder237m_layer", dict(B=2, H=4, H_kv=1, T=300, seed=74)),
    ("gpt12m_layer", dict(B=1, H=2, T=129, seed=75)),
]


def _run(w, save):
    from bwd_causal_sdpa_b200 import ATTN_OK
    from bwd_causal_sdpa_b200.runner import AttnRunner

    r = AttnRunner.from_workload(w, save=save)
    r.forward()
    r.backward()
    st = r.status()
    assert st == ATTN_OK, f"device status {st}"
    return r, r.results()


@pytest.mark.parametrize("name,over", CASES, ids=[f"{n}-{i}" for i, (n, _) in enumerate(CASES)])
def test_saved_pair_matches_oracle_and_plain_calls(name, over):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    w = make_workload(config_by_name(name), **over)
    r, got = _run(w, save=True)
    assert r.saved is not None and r.saved_bytes > 0  # bf16 with RoPE: operands kept
    errs = compare(w, got, oracle_outputs(w))
    _, plain = _run(w, save=False)
    for key in ("o", "lse"):
        assert np.array_equal(got[key], plain[key]), f"{key} differs from the plain calls"
    for key in ("dq", "dk", "dv"):
        a, b = got[key], plain[key]
        step = np.maximum(np.abs(a), np.abs(b)) * 2.0 ** -7  # one bf16 step at that magnitude
        assert np.all(np.abs(a - b) <= step + 1e-30), f"{key} differs from the plain calls"
    print(name, over, errs)
