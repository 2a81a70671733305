"""fp64 CPU oracle for Loki sparse decode-step attention.

TEST INFRASTRUCTURE.  This module exists to check the CUDA path; it is not part
of the product.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import or run it.  It shares no code with the CUDA path
and imports nothing from the product package.

What it computes, step by step, in the order the pages give:

  "PCA-project queries and keys, rank tokens using only the top-d principal
  dimensions, then compute exact attention on the top-k tokens without deleting
  any cache entries."  (paraphrase of "Loki: Low-rank Keys for Efficient Sparse
  Attention", atlas.scime.ai summary, section "Approach"; the PCA basis is
  "calibrated offline", same page, summary paragraph; the arXiv record on
  mlsanity.com, 2406.02542, "Abstract", says tokens are ranked and selected by
  attention scores computed in the low-dimensional space.)

Everything is float64.  Inputs in bf16 or fp32 are widened exactly to fp64 by
the caller; P is the fp32 basis that the GPU also receives, widened exactly.

Readings where the pages are silent (each is also listed in the design notes):
  * d = floor(d_f * D), k = floor(k_f * S), clamped to [1, D] and [1, S]
    (the caller passes the integers).
  * The ranking score is the raw low-rank dot product, without scale or softmax
    (a positive scale and a monotone map change no order).
  * Ties between equal scores go to the lower token index; the selected index
    set is reported in ascending order.
  * With grouped-query attention, the score of a key for KV head g is the sum
    over the group's query heads of their low-rank scores.
  * Exact attention uses the full D dimensions of the rotated query and the
    rotated cached key, with softmax scale 1/sqrt(D) unless given.
  * The rotated key is rounded to the cache dtype (round to nearest even) when
    it is written into the cache; values are stored unrotated.

Pins (tests/test_oracle_pins.py): every public function below is checked against
something other than itself (closed forms, brute force, a library routine for a
special case, or invariants of the definition).  No function is parity unpinned.
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np

BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


# --------------------------------------------------------------------------
# rounding to the cache dtype
# --------------------------------------------------------------------------
def round_bf16(x) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 value, ties to even.

    bfloat16 keeps 8 significant bits and the fp32 exponent range.  For
    x = m * 2^e with 0.5 <= |m| < 1 the spacing of bf16 values is 2^(e-8); below
    the smallest normal (2^-126) the spacing is fixed at 2^-133.  Results beyond
    the largest finite value become +-inf.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    q = np.maximum(e.astype(np.int64) - 8, -133)
    with np.errstate(over="ignore", invalid="ignore"):
        r = np.ldexp(np.rint(np.ldexp(x, -q)), q)
        r = np.where(np.abs(r) > BF16_MAX, np.copysign(np.inf, x), r)
    return r


def round_to_dtype(x, dtype: str) -> np.ndarray:
    """Round fp64 values to the cache dtype ("f32", "bf16") and widen back.
    dtype "f64" leaves the values untouched (used by invariance checks)."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f64":
        return x.copy()
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        return round_bf16(x)
    raise ValueError(dtype)


# --------------------------------------------------------------------------
# offline calibration: PCA of the keys
# --------------------------------------------------------------------------
def pca_basis(calib_keys) -> tuple:
    """Principal directions of a calibration batch of keys.

    Covariance C = (1/N) sum (k - mean)(k - mean)^T; its eigenvectors, sorted by
    descending eigenvalue, are the columns of P (P[:, j] is the j-th principal
    direction).  The sign of each column is fixed so that its entry of largest
    magnitude is positive.  The eigen-decomposition is a library step
    (numpy.linalg.eigh).  Returns (P [D, D], eigenvalues [D] descending).
    """
    X = np.asarray(calib_keys, dtype=np.float64)
    N, D = X.shape
    mu = X.mean(axis=0)
    Xc = X - mu[None, :]
    C = (Xc.T @ Xc) / N
    w, V = np.linalg.eigh(C)
    order = np.argsort(-w, kind="stable")
    w = w[order]
    V = V[:, order]
    lead = np.argmax(np.abs(V), axis=0)
    signs = np.sign(V[lead, np.arange(D)])
    signs[signs == 0] = 1.0
    return np.ascontiguousarray(V * signs[None, :]), w


# --------------------------------------------------------------------------
# cache append: rotate new keys into the PCA basis
# --------------------------------------------------------------------------
def rotate_keys(k_new, P, dtype: str) -> np.ndarray:
    """k_hat = k_new . P_g for every (batch, KV head, token), rounded to the
    cache dtype.  k_new: [B, Hkv, n, D]; P: [Hkv, D, D]."""
    k_new = np.asarray(k_new, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    out = np.empty_like(k_new)
    for g in range(k_new.shape[1]):
        out[:, g] = k_new[:, g] @ P[g]
    return round_to_dtype(out, dtype)


def append(K_hat, V_cache, pos: int, k_new, v_new, P, dtype: str) -> None:
    """Write the rotated new keys and the unrotated new values at positions
    [pos, pos + n) of every (batch, KV head) row, in place.  Entries below pos
    are never touched: nothing is evicted."""
    n = k_new.shape[2]
    K_hat[:, :, pos:pos + n] = rotate_keys(k_new, P, dtype)
    V_cache[:, :, pos:pos + n] = np.asarray(v_new, dtype=np.float64)


# --------------------------------------------------------------------------
# decode step
# --------------------------------------------------------------------------
def rotate_queries(q, P) -> np.ndarray:
    """q_hat_h = q_h . P_g with g the KV head of query head h.
    q: [B, Hq, D], P: [Hkv, D, D] -> [B, Hq, D]."""
    q = np.asarray(q, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    B, Hq, D = q.shape
    Hkv = P.shape[0]
    G = Hq // Hkv
    out = np.empty_like(q)
    for h in range(Hq):
        out[:, h] = q[:, h] @ P[h // G]
    return out


def lowrank_scores(q_hat, K_hat, S: int, d: int) -> np.ndarray:
    """Selection score of every cached token of every (batch, KV head) row:
    the sum over the query heads of the group of q_hat_h[:d] . k_hat[:d].
    q_hat: [B, Hq, D], K_hat: [B, Hkv, S_cap, D] -> [B, Hkv, S]."""
    B, Hq, D = q_hat.shape
    Hkv = K_hat.shape[1]
    G = Hq // Hkv
    s = np.zeros((B, Hkv, S))
    for b in range(B):
        for g in range(Hkv):
            Kd = K_hat[b, g, :S, :d]
            for h in range(g * G, (g + 1) * G):
                s[b, g] += Kd @ q_hat[b, h, :d]
    return s


def select_topk(scores, k: int) -> np.ndarray:
    """The k best tokens of every row: order by (score descending, index
    ascending), keep the first k, report them in ascending index order.
    scores: [..., S] -> int64 [..., k]."""
    s = np.asarray(scores, dtype=np.float64)
    S = s.shape[-1]
    flat = s.reshape(-1, S)
    out = np.empty((flat.shape[0], k), dtype=np.int64)
    pos = np.arange(S)
    for r in range(flat.shape[0]):
        order = np.lexsort((pos, -flat[r]))
        out[r] = np.sort(order[:k])
    return out.reshape(s.shape[:-1] + (k,))


def softmax_attention(qh, Krows, Vrows, scale: float):
    """Softmax attention of one query over a set of rows.
    Returns (output [D], weights [n])."""
    a = scale * (Krows @ qh)
    m = a.max()
    w = np.exp(a - m)
    w = w / w.sum()
    return w @ Vrows, w


def sparse_attention(q_hat, K_hat, V_cache, idx, scale: float, return_weights: bool = False):
    """Exact attention of every query head over the selected rows of its KV
    head, using the full D dimensions.  idx: [B, Hkv, k] -> out [B, Hq, D]."""
    B, Hq, D = q_hat.shape
    Hkv = K_hat.shape[1]
    G = Hq // Hkv
    out = np.empty((B, Hq, D))
    weights = np.empty((B, Hq, idx.shape[-1]))
    for b in range(B):
        for g in range(Hkv):
            rows = idx[b, g]
            Kr = K_hat[b, g, rows]
            Vr = V_cache[b, g, rows]
            for h in range(g * G, (g + 1) * G):
                out[b, h], weights[b, h] = softmax_attention(q_hat[b, h], Kr, Vr, scale)
    return (out, weights) if return_weights else out


def topk_jaccard(idx_a, idx_b) -> np.ndarray:
    """Agreement of two top-k selections, the measure the summary page reports
    between Loki and exact attention ("Key results", "Experimental setup"):
    |A n B| / |A u B| of the index sets of every row.  [..., k] -> [...]."""
    a = np.asarray(idx_a)
    b = np.asarray(idx_b)
    k = a.shape[-1]
    fa = a.reshape(-1, k)
    fb = b.reshape(-1, b.shape[-1])
    out = np.empty(fa.shape[0])
    for r in range(fa.shape[0]):
        sa, sb = set(fa[r].tolist()), set(fb[r].tolist())
        out[r] = len(sa & sb) / len(sa | sb)
    return out.reshape(a.shape[:-1])


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


def loki_decode(q, K_hat, V_cache, P, seq_len: int, d: int, k: int,
                scale: Optional[float] = None) -> Dict[str, np.ndarray]:
    """One Loki decode step over the first seq_len cached tokens.

    q: [B, Hq, D] (unrotated), K_hat: [B, Hkv, S_cap, D] rotated keys,
    V_cache: [B, Hkv, S_cap, D], P: [Hkv, D, D].
    Returns dict(out [B, Hq, D], idx [B, Hkv, k] ascending, scores [B, Hkv, S],
    q_hat [B, Hq, D], weights [B, Hq, k]).
    """
    D = np.asarray(q).shape[-1]
    if not (1 <= d <= D and 1 <= k <= seq_len):
        raise ValueError("need 1 <= d <= D and 1 <= k <= seq_len")
    sc = default_scale(D) if scale is None else float(scale)
    q_hat = rotate_queries(q, P)
    K_hat = np.asarray(K_hat, dtype=np.float64)
    V_cache = np.asarray(V_cache, dtype=np.float64)
    s = lowrank_scores(q_hat, K_hat, seq_len, d)
    idx = select_topk(s, k)
    out, w = sparse_attention(q_hat, K_hat, V_cache, idx, sc, return_weights=True)
    return dict(out=out, idx=idx, scores=s, q_hat=q_hat, weights=w)


def dense_decode(q, K_hat, V_cache, P, seq_len: int, scale: Optional[float] = None) -> np.ndarray:
    """Full attention over all seq_len cached tokens of the rotated cache
    (the "Full Attention" baseline of the summary page, section
    "Experimental setup")."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    Hkv = np.asarray(P).shape[0]
    sc = default_scale(D) if scale is None else float(scale)
    q_hat = rotate_queries(q, P)
    idx = np.broadcast_to(np.arange(seq_len), (B, Hkv, seq_len))
    return sparse_attention(q_hat, np.asarray(K_hat, dtype=np.float64),
                            np.asarray(V_cache, dtype=np.float64), idx, sc)
