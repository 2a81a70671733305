"""fp64 CPU oracle (test infrastructure only; see loki_oracle.py)."""
from .loki_oracle import (  # noqa: F401
    BF16_MAX,
    round_bf16,
    round_to_dtype,
    pca_basis,
    rotate_keys,
    append,
    rotate_queries,
    lowrank_scores,
    select_topk,
    softmax_attention,
    sparse_attention,
    default_scale,
    loki_decode,
    dense_decode,
    topk_jaccard,
)
