"""Python binding of the Loki decode-step library.

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, then their device pointers and the current CUDA stream are passed
to libloki.so.  Every step of the computation runs in the library's CUDA
kernels; PyTorch provides device memory and streams.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import torch

from . import _lib

_DTYPES = {torch.float32: _lib.LOKI_F32, torch.bfloat16: _lib.LOKI_BF16}


def _stream_ptr(device: torch.device, stream: Optional[torch.cuda.Stream]) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape: Tuple[int, ...], device: torch.device) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


class LokiCache:
    """A rotated-key KV cache in device memory: k_hat and v of shape
    [B, Hkv, capacity, D].  Keys are stored already rotated into the PCA basis;
    nothing is ever evicted.

    ``lowrank_dim`` (or an explicit ``k_lr`` of shape [B, Hkv, capacity, d_lr])
    adds the low-rank key plane: a contiguous copy of the first d_lr dims of
    every key, kept by every append, from which decodes with d <= d_lr stream
    their scores (same results, fewer HBM lines read when d_lr * element size
    is below 128 bytes)."""

    def __init__(self, batch: int, n_kv_heads: int, head_dim: int, capacity: int,
                 dtype: torch.dtype = torch.bfloat16, device=None,
                 k_hat: Optional[torch.Tensor] = None, v: Optional[torch.Tensor] = None,
                 lowrank_dim: Optional[int] = None, k_lr: Optional[torch.Tensor] = None):
        if dtype not in _DTYPES:
            raise ValueError(f"cache dtype must be float32 or bfloat16, got {dtype}")
        device = torch.device(device if device is not None else "cuda")
        if device.type != "cuda":
            raise ValueError("the cache must live in CUDA device memory")
        if device.index is None:
            device = torch.device("cuda", torch.cuda.current_device())
        shape = (batch, n_kv_heads, capacity, head_dim)
        self.k_hat = k_hat if k_hat is not None else torch.empty(shape, dtype=dtype, device=device)
        self.v = v if v is not None else torch.empty(shape, dtype=dtype, device=device)
        _need(self.k_hat, "k_hat", dtype, shape, device)
        _need(self.v, "v", dtype, shape, device)
        self.batch, self.n_kv_heads, self.head_dim, self.capacity = batch, n_kv_heads, head_dim, capacity
        self.dtype = dtype
        self.device = device
        if k_lr is not None:
            lowrank_dim = k_lr.shape[-1] if k_lr.dim() == 4 else -1
        self.d_lr = int(lowrank_dim) if lowrank_dim else 0
        if self.d_lr:
            lshape = (batch, n_kv_heads, capacity, self.d_lr)
            self.k_lr = k_lr if k_lr is not None else torch.empty(lshape, dtype=dtype, device=device)
            _need(self.k_lr, "k_lr", dtype, lshape, device)
        else:
            self.k_lr = None
        self._desc = _lib.loki_cache(_DTYPES[dtype], batch, n_kv_heads, head_dim, capacity,
                                     self.k_hat.data_ptr(), self.v.data_ptr(),
                                     self.k_lr.data_ptr() if self.k_lr is not None else None, self.d_lr)

    def desc(self) -> ctypes.POINTER(_lib.loki_cache):
        return ctypes.byref(self._desc)

    def workspace(self, seq_len: int, n_q_heads: int) -> torch.Tensor:
        """The decode workspace of this cache (scratch; no initialisation
        needed), grown when a call needs more."""
        need = loki_decode_workspace_size(self, seq_len, n_q_heads)
        ws = getattr(self, "_ws", None)
        if ws is None or ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self._ws


def loki_append(cache: LokiCache, pos: int, k_new: torch.Tensor, v_new: torch.Tensor, P: torch.Tensor,
                stream: Optional[torch.cuda.Stream] = None) -> None:
    """Rotate k_new [B, Hkv, n_new, D] by P [Hkv, D, D] (fp32) and append it with
    v_new at positions [pos, pos + n_new)."""
    n_new = k_new.shape[2] if k_new.dim() == 4 else -1
    shp = (cache.batch, cache.n_kv_heads, n_new, cache.head_dim)
    _need(k_new, "k_new", cache.dtype, shp, cache.device)
    _need(v_new, "v_new", cache.dtype, shp, cache.device)
    _need(P, "P", torch.float32, (cache.n_kv_heads, cache.head_dim, cache.head_dim), cache.device)
    _lib.check(_lib.load().loki_append(cache.desc(), int(pos), int(n_new), _ptr(k_new), _ptr(v_new), _ptr(P),
                                       _stream_ptr(cache.device, stream)))


def loki_decode_workspace_size(cache: LokiCache, seq_len: int, n_q_heads: int) -> int:
    """Bytes of workspace a decode over seq_len tokens needs."""
    n = ctypes.c_size_t(0)
    _lib.check(_lib.load().loki_decode_workspace_size(cache.desc(), int(seq_len), int(n_q_heads), ctypes.byref(n)))
    return int(n.value)


def loki_decode_attention(cache: LokiCache, seq_len: int, q: torch.Tensor, P: torch.Tensor, d: int, k: int,
                          scale: float = 0.0, out: Optional[torch.Tensor] = None,
                          idx: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                          stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One Loki decode step.  q: [B, Hq, D] in the cache dtype.  Returns
    (out [B, Hq, D] fp32, idx [B, Hkv, k] int32 ascending).  `workspace`
    (uint8 scratch on the cache's device, at least loki_decode_workspace_size
    bytes) defaults to one the cache keeps."""
    B, Hq, D = q.shape if q.dim() == 3 else (-1, -1, -1)
    _need(q, "q", cache.dtype, (cache.batch, Hq, cache.head_dim), cache.device)
    _need(P, "P", torch.float32, (cache.n_kv_heads, cache.head_dim, cache.head_dim), cache.device)
    if out is None:
        out = torch.empty((cache.batch, Hq, cache.head_dim), dtype=torch.float32, device=cache.device)
    if idx is None:
        idx = torch.empty((cache.batch, cache.n_kv_heads, int(k)), dtype=torch.int32, device=cache.device)
    _need(out, "out", torch.float32, (cache.batch, Hq, cache.head_dim), cache.device)
    _need(idx, "idx", torch.int32, (cache.batch, cache.n_kv_heads, int(k)), cache.device)
    if workspace is None:
        workspace = cache.workspace(seq_len, Hq)
    if workspace.device != cache.device or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous uint8 tensor on the cache's device")
    _lib.check(_lib.load().loki_decode_attention(cache.desc(), int(seq_len), int(Hq), _ptr(q), _ptr(P), int(d),
                                                 int(k), float(scale), _ptr(out), _ptr(idx), _ptr(workspace),
                                                 int(workspace.numel()), _stream_ptr(cache.device, stream)))
    return out, idx


def loki_decode_attention_noalloc(cache: LokiCache, seq_len: int, q: torch.Tensor, P: torch.Tensor, d: int, k: int,
                                  scale: float = 0.0, out: Optional[torch.Tensor] = None,
                                  idx: Optional[torch.Tensor] = None,
                                  stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """loki_decode_attention on the library's fixed device scratch instead of
    a workspace, for callers that cannot allocate device memory on the decode
    path.  Calls on one device share that scratch: they must not overlap on
    the GPU.  Shapes beyond its 4 MiB raise LokiError (unsupported)."""
    B, Hq, D = q.shape if q.dim() == 3 else (-1, -1, -1)
    _need(q, "q", cache.dtype, (cache.batch, Hq, cache.head_dim), cache.device)
    _need(P, "P", torch.float32, (cache.n_kv_heads, cache.head_dim, cache.head_dim), cache.device)
    if out is None:
        out = torch.empty((cache.batch, Hq, cache.head_dim), dtype=torch.float32, device=cache.device)
    if idx is None:
        idx = torch.empty((cache.batch, cache.n_kv_heads, int(k)), dtype=torch.int32, device=cache.device)
    _need(out, "out", torch.float32, (cache.batch, Hq, cache.head_dim), cache.device)
    _need(idx, "idx", torch.int32, (cache.batch, cache.n_kv_heads, int(k)), cache.device)
    with torch.cuda.device(cache.device):
        _lib.check(_lib.load().loki_decode_attention_noalloc(cache.desc(), int(seq_len), int(Hq), _ptr(q), _ptr(P),
                                                             int(d), int(k), float(scale), _ptr(out), _ptr(idx),
                                                             _stream_ptr(cache.device, stream)))
    return out, idx


def dense_decode_attention(cache: LokiCache, seq_len: int, q: torch.Tensor, P: torch.Tensor, scale: float = 0.0,
                           out: Optional[torch.Tensor] = None,
                           stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Full attention over tokens [0, seq_len) of the same rotated cache."""
    B, Hq, D = q.shape if q.dim() == 3 else (-1, -1, -1)
    _need(q, "q", cache.dtype, (cache.batch, Hq, cache.head_dim), cache.device)
    _need(P, "P", torch.float32, (cache.n_kv_heads, cache.head_dim, cache.head_dim), cache.device)
    if out is None:
        out = torch.empty((cache.batch, Hq, cache.head_dim), dtype=torch.float32, device=cache.device)
    _need(out, "out", torch.float32, (cache.batch, Hq, cache.head_dim), cache.device)
    _lib.check(_lib.load().dense_decode_attention(cache.desc(), int(seq_len), int(Hq), _ptr(q), _ptr(P),
                                                  float(scale), _ptr(out), _stream_ptr(cache.device, stream)))
    return out


def _need_token(cache, k_new: torch.Tensor, v_new: torch.Tensor, B: int) -> None:
    shp = (B, cache.n_kv_heads, cache.head_dim)
    _need(k_new, "k_new", cache.dtype, shp, cache.device)
    _need(v_new, "v_new", cache.dtype, shp, cache.device)


def loki_decode_attention_append(cache: LokiCache, seq_len: int, k_new: torch.Tensor, v_new: torch.Tensor,
                                 q: torch.Tensor, P: torch.Tensor, d: int, k: int, scale: float = 0.0,
                                 out: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                                 workspace: Optional[torch.Tensor] = None,
                                 stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One generation step: write the new token (k_new rotated by P, v_new;
    both [B, Hkv, D]) at position seq_len - 1 of every row, then the Loki
    step over tokens [0, seq_len).  Returns (out, idx) as
    loki_decode_attention."""
    B, Hq, D = q.shape if q.dim() == 3 else (-1, -1, -1)
    _need(q, "q", cache.dtype, (cache.batch, Hq, cache.head_dim), cache.device)
    _need(P, "P", torch.float32, (cache.n_kv_heads, cache.head_dim, cache.head_dim), cache.device)
    _need_token(cache, k_new, v_new, cache.batch)
    if out is None:
        out = torch.empty((cache.batch, Hq, cache.head_dim), dtype=torch.float32, device=cache.device)
    if idx is None:
        idx = torch.empty((cache.batch, cache.n_kv_heads, int(k)), dtype=torch.int32, device=cache.device)
    _need(out, "out", torch.float32, (cache.batch, Hq, cache.head_dim), cache.device)
    _need(idx, "idx", torch.int32, (cache.batch, cache.n_kv_heads, int(k)), cache.device)
    if workspace is None:
        workspace = cache.workspace(seq_len, Hq)
    _lib.check(_lib.load().loki_decode_attention_append(
        cache.desc(), int(seq_len), int(Hq), _ptr(k_new), _ptr(v_new), _ptr(q), _ptr(P), int(d), int(k),
        float(scale), _ptr(out), _ptr(idx), _ptr(workspace), int(workspace.numel()),
        _stream_ptr(cache.device, stream)))
    return out, idx


def dense_decode_attention_append(cache: LokiCache, seq_len: int, k_new: torch.Tensor, v_new: torch.Tensor,
                                  q: torch.Tensor, P: torch.Tensor, scale: float = 0.0,
                                  out: Optional[torch.Tensor] = None,
                                  stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """The generation step of the full-attention baseline: append the new
    token at position seq_len - 1, then attend tokens [0, seq_len)."""
    B, Hq, D = q.shape if q.dim() == 3 else (-1, -1, -1)
    _need(q, "q", cache.dtype, (cache.batch, Hq, cache.head_dim), cache.device)
    _need(P, "P", torch.float32, (cache.n_kv_heads, cache.head_dim, cache.head_dim), cache.device)
    _need_token(cache, k_new, v_new, cache.batch)
    if out is None:
        out = torch.empty((cache.batch, Hq, cache.head_dim), dtype=torch.float32, device=cache.device)
    _need(out, "out", torch.float32, (cache.batch, Hq, cache.head_dim), cache.device)
    _lib.check(_lib.load().dense_decode_attention_append(
        cache.desc(), int(seq_len), int(Hq), _ptr(k_new), _ptr(v_new), _ptr(q), _ptr(P), float(scale), _ptr(out),
        _stream_ptr(cache.device, stream)))
    return out


def topk_jaccard(idx_a: torch.Tensor, idx_b: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Per-row Jaccard similarity of two selections [..., k] int32 (ascending
    rows, as loki_decode_attention returns them).  Returns float32 [...]: the
    agreement of Loki's selection with the exact top-k when idx_b comes from a
    call with d = D."""
    if idx_a.shape != idx_b.shape or idx_a.dim() < 1:
        raise ValueError(f"selections must have equal shapes, got {tuple(idx_a.shape)} and {tuple(idx_b.shape)}")
    k = int(idx_a.shape[-1])
    rows = idx_a.numel() // k if k else 0
    dev = idx_a.device
    for t, nm in ((idx_a, "idx_a"), (idx_b, "idx_b")):
        if t.dtype != torch.int32 or t.device != dev or not t.is_contiguous() or dev.type != "cuda":
            raise ValueError(f"{nm} must be a contiguous int32 CUDA tensor on {dev}")
    out = torch.empty(idx_a.shape[:-1], dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _lib.check(_lib.load().loki_topk_jaccard(_ptr(idx_a), _ptr(idx_b), int(rows), k, _ptr(out),
                                                 _stream_ptr(dev, stream)))
    return out


class PagedLokiCache:
    """A paged rotated-key cache: pools k_hat and v of shape
    [num_pages, Hkv, page_size, D] shared by the sequences of a batch through a
    page table (see SeqTable).  ``lowrank_dim`` (or ``k_lr``) adds a low-rank
    key plane pool [num_pages, Hkv, page_size, d_lr], as in LokiCache."""

    def __init__(self, num_pages: int, n_kv_heads: int, head_dim: int, page_size: int,
                 dtype: torch.dtype = torch.bfloat16, device=None,
                 k_hat: Optional[torch.Tensor] = None, v: Optional[torch.Tensor] = None,
                 lowrank_dim: Optional[int] = None, k_lr: Optional[torch.Tensor] = None):
        if dtype not in _DTYPES:
            raise ValueError(f"cache dtype must be float32 or bfloat16, got {dtype}")
        device = torch.device(device if device is not None else "cuda")
        if device.type != "cuda":
            raise ValueError("the cache must live in CUDA device memory")
        if device.index is None:
            device = torch.device("cuda", torch.cuda.current_device())
        shape = (num_pages, n_kv_heads, page_size, head_dim)
        self.k_hat = k_hat if k_hat is not None else torch.empty(shape, dtype=dtype, device=device)
        self.v = v if v is not None else torch.empty(shape, dtype=dtype, device=device)
        _need(self.k_hat, "k_hat", dtype, shape, device)
        _need(self.v, "v", dtype, shape, device)
        self.num_pages, self.n_kv_heads, self.head_dim, self.page_size = num_pages, n_kv_heads, head_dim, page_size
        self.dtype = dtype
        self.device = device
        if k_lr is not None:
            lowrank_dim = k_lr.shape[-1] if k_lr.dim() == 4 else -1
        self.d_lr = int(lowrank_dim) if lowrank_dim else 0
        if self.d_lr:
            lshape = (num_pages, n_kv_heads, page_size, self.d_lr)
            self.k_lr = k_lr if k_lr is not None else torch.empty(lshape, dtype=dtype, device=device)
            _need(self.k_lr, "k_lr", dtype, lshape, device)
        else:
            self.k_lr = None
        self._desc = _lib.loki_paged_cache(_DTYPES[dtype], n_kv_heads, head_dim, page_size, num_pages,
                                           self.k_hat.data_ptr(), self.v.data_ptr(),
                                           self.k_lr.data_ptr() if self.k_lr is not None else None, self.d_lr)

    def desc(self):
        return ctypes.byref(self._desc)


class SeqTable:
    """The sequences of a batch in a paged cache: block_table [B, pages_per_seq]
    int32 page ids and seq_lens [B] int32 (or None: max_seq_len everywhere),
    both on the cache's device."""

    def __init__(self, block_table: torch.Tensor, seq_lens: Optional[torch.Tensor], max_seq_len: int):
        if block_table.dim() != 2 or block_table.dtype != torch.int32 or not block_table.is_contiguous():
            raise ValueError("block_table must be a contiguous [B, pages_per_seq] int32 tensor")
        B = int(block_table.shape[0])
        if seq_lens is not None:
            _need(seq_lens, "seq_lens", torch.int32, (B,), block_table.device)
        self.block_table, self.seq_lens, self.max_seq_len = block_table, seq_lens, int(max_seq_len)
        self.batch, self.pages_per_seq = B, int(block_table.shape[1])
        self._desc = _lib.loki_seq_table(B, self.pages_per_seq, self.max_seq_len, block_table.data_ptr(),
                                         seq_lens.data_ptr() if seq_lens is not None else None)

    def desc(self):
        return ctypes.byref(self._desc)


def loki_paged_append(cache: PagedLokiCache, seqs: SeqTable, pos: torch.Tensor, k_new: torch.Tensor,
                      v_new: torch.Tensor, P: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> None:
    """Rotate k_new [B, Hkv, n_new, D] by P and write it with v_new at tokens
    pos[b] .. pos[b] + n_new - 1 of each sequence b (pos: [B] int32)."""
    n_new = k_new.shape[2] if k_new.dim() == 4 else -1
    shp = (seqs.batch, cache.n_kv_heads, n_new, cache.head_dim)
    _need(k_new, "k_new", cache.dtype, shp, cache.device)
    _need(v_new, "v_new", cache.dtype, shp, cache.device)
    _need(P, "P", torch.float32, (cache.n_kv_heads, cache.head_dim, cache.head_dim), cache.device)
    _need(pos, "pos", torch.int32, (seqs.batch,), cache.device)
    _lib.check(_lib.load().loki_paged_append(cache.desc(), seqs.desc(), _ptr(pos), int(n_new), _ptr(k_new),
                                             _ptr(v_new), _ptr(P), _stream_ptr(cache.device, stream)))


def loki_paged_decode_attention(cache: PagedLokiCache, seqs: SeqTable, q: torch.Tensor, P: torch.Tensor, d: int,
                                k_max: int, ks: Optional[torch.Tensor] = None, scale: float = 0.0,
                                out: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                                workspace: Optional[torch.Tensor] = None,
                                stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The Loki step on a paged cache with per-sequence lengths.  Returns
    (out [B, Hq, D] fp32, idx [B, Hkv, k_max] int32, -1 past each row's k)."""
    B, Hkv, D = seqs.batch, cache.n_kv_heads, cache.head_dim
    if q.dim() != 3 or q.shape[0] != B or q.shape[2] != D:
        raise ValueError(f"q must be [B={B}, Hq, D={D}], got {tuple(q.shape)}")
    Hq = int(q.shape[1])
    _need(q, "q", cache.dtype, (B, Hq, D), cache.device)
    _need(P, "P", torch.float32, (Hkv, D, D), cache.device)
    if ks is not None:
        _need(ks, "ks", torch.int32, (B,), cache.device)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=cache.device)
    if idx is None:
        idx = torch.empty((B, Hkv, int(k_max)), dtype=torch.int32, device=cache.device)
    _need(out, "out", torch.float32, (B, Hq, D), cache.device)
    _need(idx, "idx", torch.int32, (B, Hkv, int(k_max)), cache.device)
    n = ctypes.c_size_t(0)
    lib = _lib.load()
    _lib.check(lib.loki_paged_decode_workspace_size(cache.desc(), seqs.desc(), Hq, ctypes.byref(n)))
    if workspace is None or workspace.numel() * workspace.element_size() < n.value:
        workspace = torch.empty(int(n.value), dtype=torch.uint8, device=cache.device)
    _lib.check(lib.loki_paged_decode_attention(cache.desc(), seqs.desc(), Hq, _ptr(q), _ptr(P), int(d),
                                               _ptr(ks) if ks is not None else None, int(k_max), float(scale),
                                               _ptr(out), _ptr(idx), _ptr(workspace),
                                               workspace.numel() * workspace.element_size(),
                                               _stream_ptr(cache.device, stream)))
    return out, idx


def loki_paged_decode_attention_append(cache: PagedLokiCache, seqs: SeqTable, k_new: torch.Tensor,
                                       v_new: torch.Tensor, q: torch.Tensor, P: torch.Tensor, d: int, k_max: int,
                                       ks: Optional[torch.Tensor] = None, scale: float = 0.0,
                                       out: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                                       workspace: Optional[torch.Tensor] = None,
                                       stream: Optional[torch.cuda.Stream] = None
                                       ) -> Tuple[torch.Tensor, torch.Tensor]:
    """One generation step on a paged cache: sequence b's new token (k_new[b],
    v_new[b], [B, Hkv, D]) goes to its position seq_lens[b] - 1, then the Loki
    step over its seq_lens[b] tokens."""
    B, Hkv, D = seqs.batch, cache.n_kv_heads, cache.head_dim
    if q.dim() != 3 or q.shape[0] != B or q.shape[2] != D:
        raise ValueError(f"q must be [B={B}, Hq, D={D}], got {tuple(q.shape)}")
    Hq = int(q.shape[1])
    _need(q, "q", cache.dtype, (B, Hq, D), cache.device)
    _need(P, "P", torch.float32, (Hkv, D, D), cache.device)
    _need_token(cache, k_new, v_new, B)
    if ks is not None:
        _need(ks, "ks", torch.int32, (B,), cache.device)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=cache.device)
    if idx is None:
        idx = torch.empty((B, Hkv, int(k_max)), dtype=torch.int32, device=cache.device)
    _need(out, "out", torch.float32, (B, Hq, D), cache.device)
    _need(idx, "idx", torch.int32, (B, Hkv, int(k_max)), cache.device)
    n = ctypes.c_size_t(0)
    lib = _lib.load()
    _lib.check(lib.loki_paged_decode_workspace_size(cache.desc(), seqs.desc(), Hq, ctypes.byref(n)))
    if workspace is None or workspace.numel() * workspace.element_size() < n.value:
        workspace = torch.empty(int(n.value), dtype=torch.uint8, device=cache.device)
    _lib.check(lib.loki_paged_decode_attention_append(
        cache.desc(), seqs.desc(), Hq, _ptr(k_new), _ptr(v_new), _ptr(q), _ptr(P), int(d),
        _ptr(ks) if ks is not None else None, int(k_max), float(scale), _ptr(out), _ptr(idx), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream_ptr(cache.device, stream)))
    return out, idx


def dense_paged_decode_attention(cache: PagedLokiCache, seqs: SeqTable, q: torch.Tensor, P: torch.Tensor,
                                 scale: float = 0.0, out: Optional[torch.Tensor] = None,
                                 stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Full attention over each sequence's seq_lens[b] tokens of a paged cache."""
    B, D = seqs.batch, cache.head_dim
    Hq = int(q.shape[1]) if q.dim() == 3 else -1
    _need(q, "q", cache.dtype, (B, Hq, D), cache.device)
    _need(P, "P", torch.float32, (cache.n_kv_heads, D, D), cache.device)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=cache.device)
    _need(out, "out", torch.float32, (B, Hq, D), cache.device)
    _lib.check(_lib.load().dense_paged_decode_attention(cache.desc(), seqs.desc(), Hq, _ptr(q), _ptr(P),
                                                        float(scale), _ptr(out), _stream_ptr(cache.device, stream)))
    return out


def loki_pca_workspace_size(n_heads: int, head_dim: int) -> int:
    n = ctypes.c_size_t(0)
    _lib.check(_lib.load().loki_pca_workspace_size(int(n_heads), int(head_dim), ctypes.byref(n)))
    return int(n.value)


def loki_pca_calibrate(keys: torch.Tensor, stream: Optional[torch.cuda.Stream] = None,
                       workspace: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """PCA basis of each head from its calibration keys, on the GPU.

    keys: [H, N, D] fp32 or bf16 CUDA tensor.  Returns (P [H, D, D] fp32,
    eigenvalues [H, D] fp64, descending); column j of P[g] is the j-th
    principal direction, its largest-magnitude entry positive."""
    if keys.dim() != 3 or keys.device.type != "cuda" or not keys.is_contiguous():
        raise ValueError("keys must be a contiguous [H, N, D] CUDA tensor")
    if keys.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError(f"keys dtype {keys.dtype} (float32 or bfloat16)")
    H, N, D = (int(x) for x in keys.shape)
    dev = keys.device
    need = loki_pca_workspace_size(H, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    P = torch.empty((H, D, D), dtype=torch.float32, device=dev)
    w = torch.empty((H, D), dtype=torch.float64, device=dev)
    dt = _lib.LOKI_F32 if keys.dtype == torch.float32 else _lib.LOKI_BF16
    with torch.cuda.device(dev):
        _lib.check(_lib.load().loki_pca_calibrate(_ptr(keys), dt, H, N, D, _ptr(P), _ptr(w), _ptr(workspace),
                                                  workspace.numel() * workspace.element_size(),
                                                  _stream_ptr(dev, stream)))
    return P, w


def loki_decode_launch_shape(cache: LokiCache, seq_len: int, n_q_heads: int, k: int = 1,
                             dense: bool = False) -> Tuple[int, int, int, int]:
    """Grid sizes of a decode call.  Loki: (rotation CTAs, decode CTAs per row
    in one cluster, decode CTAs, 1 for the short-row kernel (rows of at most
    8192 tokens, where it fits as many CTAs per SM as the long-row kernel)
    else 0).  Dense: (0, CTAs per row in one cluster, CTAs, 0)."""
    shape = (ctypes.c_int32 * 4)()
    with torch.cuda.device(cache.device):
        _lib.check(_lib.load().loki_decode_launch_shape(cache.desc(), int(seq_len), int(n_q_heads), int(k),
                                                        int(bool(dense)), shape))
    return tuple(int(x) for x in shape)


def loki_status_string(status: int) -> str:
    return _lib.load().loki_status_string(int(status)).decode()


def loki_version() -> int:
    return int(_lib.load().loki_version())


class DecodeGraph:
    """One Loki decode step from and to pinned host memory, captured once as a
    CUDA graph and replayed: the copy of the query in (`q_host`), the decode
    kernel(s) of loki_decode_attention, and the copies of the output and the
    selected indices out (`out_host`, `idx_host`).  A replay launches the
    whole step with one graph launch instead of four launches.

    Fill `q_host` before `replay()`; read `out_host` / `idx_host` once the
    stream has passed the replay (for example after torch.cuda.synchronize()).
    The cache, seq_len, P, d and k are fixed at capture; the cache contents may
    change between replays (an append before each step, say).  `out` and `idx`
    sit back to back in one device buffer, so that one copy brings both back
    (`out_host` and `idx_host` are views of one pinned buffer).  Capture happens
    in the constructor, after one eager warm-up call (which sets the kernels'
    attributes and allocates the workspace), so the constructor must not run
    inside another capture."""

    def __init__(self, cache: LokiCache, seq_len: int, P: torch.Tensor, d: int, k: int, n_q_heads: int,
                 scale: float = 0.0):
        dev = cache.device
        self.cache, self.seq_len, self.P, self.d, self.k, self.scale = cache, int(seq_len), P, int(d), int(k), scale
        shape = (cache.batch, int(n_q_heads), cache.head_dim)
        ishape = (cache.batch, cache.n_kv_heads, self.k)
        n_out, n_idx = shape[0] * shape[1] * shape[2], ishape[0] * ishape[1] * ishape[2]
        self.q_host = torch.empty(shape, dtype=cache.dtype).pin_memory()
        self.res_host = torch.empty(n_out + n_idx, dtype=torch.float32).pin_memory()
        self.out_host = self.res_host[:n_out].view(shape)
        self.idx_host = self.res_host[n_out:].view(torch.int32).view(ishape)
        self.q = torch.zeros(shape, dtype=cache.dtype, device=dev)
        self.res = torch.empty(n_out + n_idx, dtype=torch.float32, device=dev)
        self.out = self.res[:n_out].view(shape)
        self.idx = self.res[n_out:].view(torch.int32).view(ishape)
        self.workspace = cache.workspace(self.seq_len, int(n_q_heads))
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            self._step()  # warm-up: kernel attributes, first-call lookups
        side.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=side):
            self._step()
        torch.cuda.current_stream(dev).wait_stream(side)

    def _step(self) -> None:
        self.q.copy_(self.q_host, non_blocking=True)
        loki_decode_attention(self.cache, self.seq_len, self.q, self.P, self.d, self.k, scale=self.scale,
                              out=self.out, idx=self.idx, workspace=self.workspace)
        self.res_host.copy_(self.res, non_blocking=True)

    def replay(self) -> None:
        """Enqueue the step on the current stream."""
        self.graph.replay()
