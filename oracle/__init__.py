"""CPU oracle (test infrastructure only; see ``ress_oracle``)."""

from .ress_oracle import (  # noqa: F401
    block_drift,
    block_logits,
    block_probs,
    drift_block,
    dropped_blocks,
    pool_blocks,
    select_blocks,
    selection_scores,
    sparse_attention,
    sparse_attention_block,
    topk_lowest_index,
    value_contrast,
)
