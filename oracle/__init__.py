"""Plain fp64 CPU oracle for online-softmax attention.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package. The CUDA library (``online_softmax_attention_fwd_b200``)
never imports it and shares no code, header, table or helper with it; the only thing both sides
see is the seeded input generator module, which holds no attention arithmetic.

Every function here is the plain definition written out in NumPy float64, not the blocked online
algorithm the kernels run (see ``attention.py`` for the passage each one follows).

Parity status: every public function is pinned by ``tests/test_oracle.py`` against something other
than itself (hand-worked values, closed forms, invariants, finite differences, a library attention
routine, monoid algebra). No function is "parity unpinned".
"""
from .attention import (  # noqa: F401
    visible_mask,
    attention_scores,
    attention_probs,
    attention_fwd,
    attention_fwd_rows,
    attention_bwd,
    attention_fwd_varlen,
    attention_fwd_fp8,
    e4m3_to_float,
    attention_bwd_varlen,
    decode_attention,
    decode_attention_paged,
    decode_attention_qlen,
    decode_attention_paged_qlen,
    paged_rows,
    monoid_identity,
    monoid_leaf,
    monoid_merge,
    monoid_finalize,
)
