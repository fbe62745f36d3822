"""CPU oracle for causal scaled-dot-product attention, forward and backward.

TEST INFRASTRUCTURE. This package is the slow, plain, float64 statement of
what the attention library computes. It is imported only by the tests, by the
smoke check in ``__graft_entry__`` and by the CPU-baseline leg of ``bench.py``;
the library itself never imports, links or calls anything here, and shares no
code with it (the CUDA path lives in ``bwd_causal_sdpa_b200``). Both sides take
their seeded inputs from ``workloads``, which holds no attention arithmetic.

Every function in ``oracle.attention`` is pinned by the CPU tests against
something other than itself: central finite differences, closed forms, hand
derived worked examples (``tests/golden``), invariants (softmax rows sum to 1,
causality, RoPE norm preservation and relative-position dependence,
packed-equals-separate documents) and the float64 PyTorch reference
``scaled_dot_product_attention`` on the cases it covers. ``oracle.decode``
(one new token against a key/value cache) is pinned against the last row of
the training forward, a closed form and invariants. No function here is
"parity unpinned". ``oracle.projection`` (the QKV projection with its RoPE
and head layout, the output projection, and their backward products) is
pinned against brute-force sums, finite differences and the attention
oracle's own RoPE (rotating in the projection equals rotating in the
attention).
"""

from .decode import decode_forward
from .projection import (
    out_projection,
    out_projection_backward,
    qkv_projection,
    qkv_projection_backward,
)
from .attention import (
    attention_backward,
    attention_forward,
    backward_head,
    doc_layout,
    forward_head,
    rope_angles_f64,
    rope_rotate,
    rope_rotate_inverse,
)

__all__ = [
    "decode_forward",
    "out_projection",
    "out_projection_backward",
    "qkv_projection",
    "qkv_projection_backward",
    "attention_backward",
    "attention_forward",
    "backward_head",
    "doc_layout",
    "forward_head",
    "rope_angles_f64",
    "rope_rotate",
    "rope_rotate_inverse",
]
