"""Loki sparse decode-step attention for NVIDIA B200 (sm_100a).

Keys and queries are rotated into an offline PCA basis, every cached token is
scored on its first d principal dimensions, the k best tokens of each (batch,
KV head) row are selected, and exact softmax attention runs over those rows
("Loki: Low-rank Keys for Efficient Sparse Attention", atlas.scime.ai summary,
section "Approach").  The work is done by hand-written CUDA kernels behind the
C ABI of include/loki.h (libloki.so); this package is its Python binding.
"""
from ._lib import LIB_PATH, LokiError, load as load_library
from .api import (
    DecodeGraph,
    LokiCache,
    PagedLokiCache,
    SeqTable,
    dense_decode_attention,
    dense_decode_attention_append,
    dense_paged_decode_attention,
    loki_append,
    loki_decode_attention,
    loki_decode_attention_append,
    loki_decode_attention_noalloc,
    loki_decode_launch_shape,
    loki_decode_workspace_size,
    loki_paged_append,
    loki_paged_decode_attention,
    loki_paged_decode_attention_append,
    loki_pca_calibrate,
    loki_pca_workspace_size,
    loki_status_string,
    loki_version,
    topk_jaccard,
)
from .sharding import shard_batches

__all__ = [
    "DecodeGraph",
    "LIB_PATH",
    "LokiError",
    "load_library",
    "LokiCache",
    "PagedLokiCache",
    "SeqTable",
    "loki_paged_append",
    "loki_paged_decode_attention",
    "loki_paged_decode_attention_append",
    "loki_decode_attention_append",
    "dense_decode_attention_append",
    "dense_paged_decode_attention",
    "loki_append",
    "loki_decode_attention",
    "loki_decode_attention_noalloc",
    "dense_decode_attention",
    "loki_decode_launch_shape",
    "loki_decode_workspace_size",
    "loki_pca_calibrate",
    "loki_pca_workspace_size",
    "loki_status_string",
    "loki_version",
    "topk_jaccard",
    "shard_batches",
]
