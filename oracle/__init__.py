"""CPU oracle (test infrastructure only; see ``ress_oracle``)."""

from .ress_oracle import (  # noqa: F401
    block_drift,
    block_logits,
    block_probs,
    cdf_counts,
    drift_block,
    dropped_blocks,
    pool_blocks,
    select_blocks,
    select_blocks_cdf,
    selection_scores,
    sparse_attention,
    sparse_attention_block,
    topk_lowest_index,
    value_contrast,
)
