"""Seeded random inputs for synthetic decode steps.

Two key generators stand in for real model KV caches (no weights or datasets
are available); both follow the observation on the Loki pages that keys lie in
a low-dimensional subspace ("Loki: Low-rank Keys for Efficient Sparse
Attention", atlas.scime.ai summary, section "Approach"; mlsanity.com arXiv
record 2406.02542, "Abstract"):

* ``rank8``: K = Z A + 0.05 N with Z ~ N(0,1) of shape [n, 8], A ~ N(0,1)/sqrt(8)
  of shape [8, D] fixed per KV head, and N ~ N(0,1) of shape [n, D].
* ``powerlaw``: K = mu + (Z * sqrt(lambda)) U^T with Z ~ N(0,1) [n, D], a Haar
  random orthonormal U per KV head, lambda_i = c * i^-alpha normalised so that
  sum(lambda) = D, and a per-head mean offset mu ~ N(0, mean_std^2).

Values and queries are N(0, 1).  Every array is drawn from a numpy PCG64 stream
keyed by (seed, stream id, batch index, head index), so any subset of rows can
be regenerated on its own and matches the same rows of a full draw.  Values are
then cast to the cache dtype; both the GPU path and the oracle consume those
cast values (the oracle widens them exactly to fp64).

Nothing here computes any part of the attention method.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

from .configs import Workload

# stream ids for the seed sequences
_MODEL, _CALIB, _KEYS, _VALUES, _QUERY, _NEWTOK = 1, 2, 3, 4, 5, 6


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng([int(x) for x in key])


@dataclass
class KeyModel:
    """Distribution of the keys of one KV head."""
    kind: str
    D: int
    A: Optional[np.ndarray] = None      # rank8: [8, D]
    U: Optional[np.ndarray] = None      # powerlaw: [D, D] orthonormal columns
    lam: Optional[np.ndarray] = None    # powerlaw: [D] descending variances
    mu: Optional[np.ndarray] = None     # powerlaw: [D] mean offset


def haar_orthonormal(D: int, rng: np.random.Generator) -> np.ndarray:
    """Haar-distributed orthonormal matrix: QR of a Gaussian matrix with the
    signs of R's diagonal folded into Q (Mezzadri, 2007)."""
    G = rng.standard_normal((D, D))
    Q, R = np.linalg.qr(G)
    return Q * np.sign(np.diag(R))[None, :]


def power_law_spectrum(D: int, alpha: float) -> np.ndarray:
    i = np.arange(1, D + 1, dtype=np.float64)
    lam = i ** (-alpha)
    return lam * (D / lam.sum())


def make_key_model(w: Workload, g: int) -> KeyModel:
    rng = _rng(w.seed, _MODEL, g)
    D = w.head_dim
    if w.generator == "rank8":
        A = rng.standard_normal((8, D)) / np.sqrt(8.0)
        return KeyModel(kind="rank8", D=D, A=A)
    if w.generator == "powerlaw":
        U = haar_orthonormal(D, rng)
        mu = rng.standard_normal(D) * w.mean_std
        return KeyModel(kind="powerlaw", D=D, U=U, lam=power_law_spectrum(D, w.alpha), mu=mu)
    raise ValueError(f"unknown generator {w.generator!r}")


def draw_keys(model: KeyModel, n: int, rng: np.random.Generator) -> np.ndarray:
    """n keys of one head, fp64 [n, D]."""
    D = model.D
    if model.kind == "rank8":
        Z = rng.standard_normal((n, 8))
        N = rng.standard_normal((n, D))
        return Z @ model.A + 0.05 * N
    Z = rng.standard_normal((n, D))
    return model.mu[None, :] + (Z * np.sqrt(model.lam)[None, :]) @ model.U.T


def draw_normal(shape: Sequence[int], rng: np.random.Generator) -> np.ndarray:
    return rng.standard_normal(tuple(shape))


def to_cache_dtype(x: np.ndarray, dtype: str):
    """Cast fp64 values to the cache dtype.

    Returns ``(tensor, exact)``: a CPU torch tensor in the cache dtype and a
    fp64 numpy array holding exactly the same values.
    """
    import torch
    x32 = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        t = torch.from_numpy(x32.copy())
    elif dtype == "bf16":
        t = torch.from_numpy(x32).to(torch.bfloat16)
    else:
        raise ValueError(dtype)
    return t, t.to(torch.float64).numpy()


def calibration_keys(w: Workload, g: int) -> np.ndarray:
    """The calibration batch for KV head g (fp64 [n_calib, D])."""
    return draw_keys(make_key_model(w, g), w.n_calib, _rng(w.seed, _CALIB, g))


def row_keys(w: Workload, b: int, g: int, n: int, models: Optional[List[KeyModel]] = None) -> np.ndarray:
    m = models[g] if models is not None else make_key_model(w, g)
    return draw_keys(m, n, _rng(w.seed, _KEYS, b, g))


def row_values(w: Workload, b: int, g: int, n: int) -> np.ndarray:
    return draw_normal((n, w.head_dim), _rng(w.seed, _VALUES, b, g))


def queries(w: Workload, b: int, step: int = 0) -> np.ndarray:
    return draw_normal((w.n_q_heads, w.head_dim), _rng(w.seed, _QUERY, b, step))


def new_token(w: Workload, b: int, step: int, models: Optional[List[KeyModel]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Key and value of the token appended at generation step ``step`` for
    batch b: fp64 arrays [Hkv, D] each."""
    ks, vs = [], []
    for g in range(w.n_kv_heads):
        m = models[g] if models is not None else make_key_model(w, g)
        rng = _rng(w.seed, _NEWTOK, b, g, step)
        ks.append(draw_keys(m, 1, rng)[0])
        vs.append(rng.standard_normal(w.head_dim))
    return np.stack(ks), np.stack(vs)


def decode_inputs(w: Workload, seq_len: Optional[int] = None,
                  batches: Optional[Iterable[int]] = None) -> Dict[str, object]:
    """Host inputs of one decode step, already cast to the cache dtype.

    Returns a dict with torch CPU tensors ``keys`` and ``values`` of shape
    [B', Hkv, S, D] (keys NOT yet rotated), ``q`` [B', Hq, D], the matching fp64
    numpy arrays ``keys64``, ``values64``, ``q64``, and ``calib`` (list over KV
    heads of fp64 [n_calib, D] calibration batches).  ``batches`` selects a subset
    of batch indices (default: all); rows are generated independently, so a
    subset equals the same rows of the full draw.
    """
    import torch
    S = w.seq_len if seq_len is None else seq_len
    bs = list(range(w.batch)) if batches is None else list(batches)
    models = [make_key_model(w, g) for g in range(w.n_kv_heads)]
    K = np.empty((len(bs), w.n_kv_heads, S, w.head_dim))
    V = np.empty_like(K)
    Q = np.empty((len(bs), w.n_q_heads, w.head_dim))
    for i, b in enumerate(bs):
        for g in range(w.n_kv_heads):
            K[i, g] = row_keys(w, b, g, S, models)
            V[i, g] = row_values(w, b, g, S)
        Q[i] = queries(w, b)
    kt, k64 = to_cache_dtype(K, w.dtype)
    vt, v64 = to_cache_dtype(V, w.dtype)
    qt, q64 = to_cache_dtype(Q, w.dtype)
    calib = [calibration_keys(w, g) for g in range(w.n_kv_heads)]
    return dict(keys=kt, values=vt, q=qt, keys64=k64, values64=v64, q64=q64,
                calib=calib, batches=bs, seq_len=S)


def device_keys(model: KeyModel, batch: int, n: int, gen, device, dtype) -> "torch.Tensor":
    """Keys of one KV head for a whole batch drawn on the GPU: the same
    distribution as draw_keys with torch's generator `gen` (so not the same
    numbers).  Returns [batch, n, D] in the torch dtype `dtype`.  Used to fill
    large caches quickly; rows checked against the oracle are overwritten with
    host draws."""
    import torch
    D = model.D
    if model.kind == "rank8":
        A = torch.as_tensor(model.A, dtype=torch.float32, device=device)
        Z = torch.randn((batch, n, 8), generator=gen, device=device)
        N = torch.randn((batch, n, D), generator=gen, device=device)
        return (Z @ A + 0.05 * N).to(dtype)
    U = torch.as_tensor(model.U, dtype=torch.float32, device=device)
    sl = torch.as_tensor(np.sqrt(model.lam), dtype=torch.float32, device=device)
    mu = torch.as_tensor(model.mu, dtype=torch.float32, device=device)
    out = torch.empty((batch, n, D), dtype=dtype, device=device)
    step = max(1, (1 << 24) // max(1, n * D))   # bound the fp32 temporaries
    for b0 in range(0, batch, step):
        Z = torch.randn((min(step, batch - b0), n, D), generator=gen, device=device)
        out[b0:b0 + Z.shape[0]] = (mu + (Z * sl) @ U.T).to(dtype)
    return out
