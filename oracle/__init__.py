"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``; never by the library.
"""

from .attention import (  # noqa: F401
    attention_bwd_gqa_ref,
    attention_bwd_ref,
    attention_fwd_gqa_ref,
    attention_fwd_ref,
    attention_rows_ref,
    e4m3_p_rounding_bound,
    online_softmax_attention,
    safe_softmax,
    scores,
    softmax_merge,
)
