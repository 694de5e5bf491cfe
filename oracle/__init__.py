"""CPU oracle (test infrastructure only; see ``ress_oracle``)."""

from .ress_oracle import (  # noqa: F401
    block_drift,
    block_logits,
    block_probs,
    cdf_counts,
    drift_block,
    drift_layout_block,
    dropped_blocks,
    pool_blocks,
    pool_blocks_valid,
    select_blocks,
    select_blocks_cdf,
    select_blocks_layout,
    selection_scores,
    sparse_attention,
    sparse_attention_block,
    sparse_attention_layout_block,
    topk_lowest_index,
    value_contrast,
    view_layout,
)
