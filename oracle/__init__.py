"""fp64 CPU oracle for exact attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs may import this package.  The product path never does.
"""

from .attention import (  # noqa: F401
    attention_forward,
    attention_forward_fp8,
    attention_head,
    attention_rows,
    attention_scores,
    block_keep,
    fp8_e4m3_decode,
    gather_paged_kv,
    gqa_kv_head,
    paged_append,
    paged_decode,
    paged_prefill,
    softmax_with_lse,
)
