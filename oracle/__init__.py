"""Float64 CPU oracle for hybrid Top-k+Top-p block-sparse attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. The CUDA library never calls it and shares no code with it.
"""

from .spa2_oracle import (  # noqa: F401
    block_counts,
    pool_blocks,
    pooled_attention,
    topk_count,
    topp_count,
    select_row,
    select_blocks,
    block_mask,
    token_mask,
    masked_attn_fwd,
    masked_attn_fwd_rows,
    masked_attn_bwd,
    masked_attn_bwd_blocks,
    masked_attn_bwd_rows,
    attn_flops,
)
