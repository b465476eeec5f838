"""fp64 CPU oracle for tiled attention — test infrastructure only.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg use it;
the CUDA library never imports it.
"""
from .attention_oracle import (  # noqa: F401
    attention_backward,
    attention_backward_block,
    attention_backward_sampled,
    attention_forward,
    attention_forward_block,
    attention_forward_blocked,
    attention_forward_kv,
    attention_forward_rows,
    attention_rows_fwd_bwd,
    head_row_stats,
    kv_head_of,
    merge_partials,
    probs,
    row_lse,
    scores,
)
