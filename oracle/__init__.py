"""Float64 CPU oracle of the S3R decode step: test infrastructure only.

Only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
"""
from .s3r_oracle import (  # noqa: F401
    NEG_INF, attend, dense_decode, inverse_cdf, kv_append, kv_rollback, page_scores, page_summaries,
    paged_attention, residual_weights, sample_rows, select_top_pages, softmax_t, sparse_draft_attn,
    sparse_draft_select, spec_sample, verify_attn, node_budget, tree_ancestor_masks, tree_verify_attn,
    tree_spec_sample, chain_parents, build_tree,
)
