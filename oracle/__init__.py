"""Float64 CPU oracle for gated block-sparse causal attention.

TEST INFRASTRUCTURE: imported only by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline / reference arm of ``bench.py``. The CUDA library never
imports it and it never imports the CUDA library.
"""
from .gated_attention import (  # noqa: F401
    SPARSE,
    THRESHOLD,
    TRAIN,
    attended_blocks,
    attended_pairs,
    gated_attention_backward,
    gated_attention_forward,
    gated_attention_naive,
    gated_decode,
    gated_decode_paged,
    log_gates,
    select_blocks,
    threshold_count,
)
