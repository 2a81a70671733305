"""Workload shapes for synthetic decode steps.

The shapes follow the models and settings that the Loki summary page
("Loki: Low-rank Keys for Efficient Sparse Attention", atlas.scime.ai,
sections "Key results" and "Measured effects reported in the paper") evaluates:
Llama2-7B, Llama2-13B at prompt 3072 + generation 512, Llama3-8B and
Mistral-7B, with key budget k_f and reduced dimension d_f drawn from
{0.125, 0.25, 0.5}.  No model weights or datasets are used: keys come from
seeded generators whose PCA spectrum is low rank or power law.

Integer sizes from fractions: d = floor(d_f * D) and k = floor(k_f * S), each
clamped to [1, D] and [1, S].
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional

BASE_SEED = 20240604


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str            # "f32" or "bf16": dtype of the cache, queries and new keys/values
    batch: int            # B
    n_q_heads: int        # Hq
    n_kv_heads: int       # Hkv
    head_dim: int         # D
    seq_len: int          # S, cache length attended by the decode step
    d_f: float
    k_f: float
    generator: str        # "rank8" (low rank + noise) or "powerlaw"
    alpha: float = 1.5    # power-law exponent of the key spectrum
    mean_std: float = 0.5 # std of the per-head key mean offset (power-law generator)
    n_calib: int = 8192   # calibration keys per KV head for the offline PCA
    seed: int = BASE_SEED
    prompt_len: Optional[int] = None   # generation workloads: prompt cache length
    gen_steps: Optional[int] = None    # generation workloads: decode steps

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def d(self) -> int:
        return reduced_dim(self.d_f, self.head_dim)

    @property
    def k(self) -> int:
        return key_budget(self.k_f, self.seq_len)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def rows(self) -> int:
        return self.batch * self.n_kv_heads

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    def loki_bytes(self) -> int:
        """Algorithmic HBM bytes of one sparse decode step: S*d*e low-rank key
        bytes plus k*2D*e gathered key/value bytes, per (batch, KV head)."""
        e = self.elem_bytes
        per_row = self.seq_len * self.d * e + self.k * 2 * self.head_dim * e
        return self.rows * per_row

    def dense_bytes(self) -> int:
        e = self.elem_bytes
        return self.rows * self.seq_len * 2 * self.head_dim * e


def reduced_dim(d_f: float, D: int) -> int:
    return max(1, min(D, int(math.floor(d_f * D + 1e-9))))


def key_budget(k_f: float, S: int) -> int:
    return max(1, min(S, int(math.floor(k_f * S + 1e-9))))


WORKLOADS: Dict[str, Workload] = {
    # tiny fp32 case: B1, 2 heads, D64, S256, d16, k64; keys are rank 8 plus noise
    "tiny-fp32": Workload(
        name="tiny-fp32", dtype="f32", batch=1, n_q_heads=2, n_kv_heads=2,
        head_dim=64, seq_len=256, d_f=0.25, k_f=0.25, generator="rank8",
        n_calib=512, seed=BASE_SEED + 0),
    # Llama2-7B-like decode, one layer: B1, 32 MHA heads, D128, S4096
    "llama2-7b-decode": Workload(
        name="llama2-7b-decode", dtype="bf16", batch=1, n_q_heads=32, n_kv_heads=32,
        head_dim=128, seq_len=4096, d_f=0.25, k_f=0.25, generator="powerlaw",
        alpha=1.5, n_calib=8192, seed=BASE_SEED + 1),
    # Llama2-13B-like generation, one layer: B16, 40 heads, prompt 3072 then 512 steps.
    # seq_len is the last step's length; each step t attends over prompt_len + t + 1.
    "llama2-13b-generation": Workload(
        name="llama2-13b-generation", dtype="bf16", batch=16, n_q_heads=40, n_kv_heads=40,
        head_dim=128, seq_len=3584, d_f=0.25, k_f=0.25, generator="powerlaw",
        alpha=1.5, n_calib=8192, seed=BASE_SEED + 2, prompt_len=3072, gen_steps=512),
    # Llama3-8B-like GQA decode: B8, 32 query heads over 8 KV heads, S32768
    "llama3-8b-gqa-decode": Workload(
        name="llama3-8b-gqa-decode", dtype="bf16", batch=8, n_q_heads=32, n_kv_heads=8,
        head_dim=128, seq_len=32768, d_f=0.5, k_f=0.125, generator="powerlaw",
        alpha=1.2, n_calib=8192, seed=BASE_SEED + 3),
}

MISTRAL_SEQ = (4096, 16384, 65536, 131072)
MISTRAL_BATCH = (1, 8, 32, 64)
MISTRAL_FRACS = (0.125, 0.25, 0.5)


def mistral_sweep_points() -> List[Workload]:
    """Mistral-7B-like GQA sweep: 32 query / 8 KV heads, D128, every
    (S, B, d_f, k_f) combination; 144 points."""
    pts = []
    for S in MISTRAL_SEQ:
        for B in MISTRAL_BATCH:
            for d_f in MISTRAL_FRACS:
                for k_f in MISTRAL_FRACS:
                    pts.append(Workload(
                        name=f"mistral-7b-gqa-s{S}-b{B}-d{d_f}-k{k_f}", dtype="bf16",
                        batch=B, n_q_heads=32, n_kv_heads=8, head_dim=128, seq_len=S,
                        d_f=d_f, k_f=k_f, generator="powerlaw", alpha=1.5,
                        n_calib=8192, seed=BASE_SEED + 4))
    return pts


def get_workload(name: str) -> Workload:
    if name in WORKLOADS:
        return WORKLOADS[name]
    for w in mistral_sweep_points():
        if w.name == name:
            return w
    raise KeyError(f"unknown workload {name!r}; known: {sorted(WORKLOADS)} + mistral sweep")
