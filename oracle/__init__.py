"""fp64 CPU oracle (test infrastructure; see dsa_oracle's header)."""
from .dsa_oracle import (attended_pairs, bf16_to_f64, block_scores, block_weights,  # noqa: F401
                         block_probabilities, decode, dense_pairs, forced_set, forward, group_scores,
                         kept_keys, pool_blocks, row_width, select_blocks, select_blocks_group,
                         select_blocks_threshold, sparse_attention,
                         sparse_attention_backward)
