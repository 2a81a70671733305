"""Comparison rules between the CUDA path and the fp64 oracle.

Selection.  The GPU ranks tokens by fp32 scores, the oracle by fp64 scores, so
keys whose scores are (nearly) tied with the k-th best may legitimately swap.
Rule: let s_k be the oracle's k-th best score and tau = 1e-4 * max(|s_k|,
rms(s)) (the relative tie band of 1e-4 around the k-th score, with an rms floor
for s_k near 0).  Keys with |s_i - s_k| <= tau form the tie band.  The GPU set
must have exactly k distinct indices in [0, S), ascending; it must contain
every oracle-selected key outside the band and no unselected key outside the
band.

Output.  When the GPU set equals the oracle's set, the GPU output is compared
with the oracle's output.  When it differs by tie-band swaps only, it is one of
several valid selections; the attention output is then uniquely determined by
that selection, and the oracle computes it from its own inputs over that set.

Tolerances: 1e-4 absolute for fp32 inputs, 5e-3 absolute for bf16 inputs
(fp32 accumulation on the GPU).
"""
from __future__ import annotations

import numpy as np

import oracle

TOL = {"f32": 1e-4, "bf16": 5e-3}
TIE_REL = 1e-4


def tie_band(scores_row: np.ndarray, k: int):
    s = np.asarray(scores_row, dtype=np.float64)
    order = np.lexsort((np.arange(len(s)), -s))
    sk = s[order[k - 1]]
    tau = TIE_REL * max(abs(sk), float(np.sqrt(np.mean(s * s))))
    return sk, tau


def check_selection(gpu_idx_row, scores_row, k: int, oracle_idx_row=None) -> str:
    """'' if the GPU selection is valid under the tie-band rule, else a message."""
    g = np.asarray(gpu_idx_row, dtype=np.int64)
    s = np.asarray(scores_row, dtype=np.float64)
    S = len(s)
    if g.shape != (k,):
        return f"expected {k} indices, got shape {g.shape}"
    if np.any(g < 0) or np.any(g >= S):
        return f"index out of range [0, {S}): min {g.min()} max {g.max()}"
    if np.any(np.diff(g) <= 0):
        return "indices not strictly ascending (duplicate or unordered)"
    o = oracle.select_topk(s[None], k)[0] if oracle_idx_row is None else np.asarray(oracle_idx_row)
    if np.array_equal(g, o):
        return ""
    sk, tau = tie_band(s, k)
    band = np.abs(s - sk) <= tau
    gs, os_ = set(g.tolist()), set(o.tolist())
    missing = [i for i in os_ - gs if not band[i]]
    extra = [i for i in gs - os_ if not band[i]]
    if missing or extra:
        return (f"selection differs outside the tie band (s_k={sk:.6g}, tau={tau:.3g}): "
                f"missing {missing[:8]} (scores {s[missing[:8]]}), extra {extra[:8]} (scores {s[extra[:8]]})")
    return ""


def check_decode(gpu_out, gpu_idx, ref: dict, q_hat, K_hat, V, scale: float, dtype: str,
                 rows=None) -> dict:
    """Compare one decode step.  ref: oracle.loki_decode result.  rows: optional
    list of (b, g) pairs to check (default: all).  Returns stats; raises
    AssertionError on a violation."""
    B, Hq, D = gpu_out.shape
    Hkv = gpu_idx.shape[1]
    G = Hq // Hkv
    k = gpu_idx.shape[2]
    tol = TOL[dtype]
    if rows is None:
        rows = [(b, g) for b in range(B) for g in range(Hkv)]
    stats = dict(rows=0, swapped_rows=0, max_err=0.0)
    for (b, g) in rows:
        msg = check_selection(gpu_idx[b, g], ref["scores"][b, g], k, ref["idx"][b, g])
        assert not msg, f"row (b={b}, g={g}): {msg}"
        same = np.array_equal(np.asarray(gpu_idx[b, g]), ref["idx"][b, g])
        for h in range(g * G, (g + 1) * G):
            if same:
                expect = ref["out"][b, h]
            else:
                sel = np.asarray(gpu_idx[b, g], dtype=np.int64)
                expect, _ = oracle.softmax_attention(q_hat[b, h], K_hat[b, g, sel], V[b, g, sel], scale)
            err = float(np.max(np.abs(np.asarray(gpu_out[b, h], dtype=np.float64) - expect)))
            stats["max_err"] = max(stats["max_err"], err)
            assert err <= tol, f"row (b={b}, g={g}) head {h}: max |gpu - oracle| = {err:.3g} > {tol}"
        stats["rows"] += 1
        stats["swapped_rows"] += 0 if same else 1
    return stats


def check_dense(gpu_out, ref_out, dtype: str, heads=None) -> float:
    tol = TOL[dtype]
    g = np.asarray(gpu_out, dtype=np.float64)
    r = np.asarray(ref_out, dtype=np.float64)
    if heads is not None:
        g = np.stack([g[b, h] for b, h in heads])
        r = np.stack([r[b, h] for b, h in heads])
    err = float(np.max(np.abs(g - r)))
    assert err <= tol, f"dense: max |gpu - oracle| = {err:.3g} > {tol}"
    return err


def gamma(n: int) -> float:
    u = 2.0 ** -24
    return n * u / (1 - n * u)


def check_append(gpu_khat, keys64, P64, dtype: str, tensor_core: bool = False) -> dict:
    """GPU rotated keys vs exact fp64 rotation.  The GPU accumulates the D
    products in fp32 and rounds once to the cache dtype.  With
    bound = gamma_D * sum_i |k_i P_ij| (the fp32 dot-product error bound), the
    fp32 value y satisfies |y - exact| <= bound, so:
      fp32 cache: |gpu - exact| <= bound;
      bf16 cache: gpu = RNE_bf16(y) lies in [RNE(exact - bound), RNE(exact + bound)]
      (RNE is monotone); where it differs from RNE(exact) that is explained by
      fp32 accumulation alone.
    tensor_core: the bulk path of bf16 caches splits P into three bf16 terms
    (their sum is P to 2^-27 relative) and accumulates the 3*D exact products
    in fp32 on the tensor cores, whose accumulation is not assumed to round to
    nearest: bound = 2 * gamma_{3D} * sum_i |k_i P_ij| (+ the split residual)."""
    D = keys64.shape[-1]
    exact = np.einsum("bgti,gij->bgtj", keys64, P64)
    mag = np.einsum("bgti,gij->bgtj", np.abs(keys64), np.abs(P64))
    if tensor_core:
        bound = (2.0 * gamma(3 * D) + 2.0 ** -26) * mag + 1e-300
    else:
        bound = gamma(D) * mag + 1e-300
    g = np.asarray(gpu_khat, dtype=np.float64)
    if dtype == "f32":
        err = np.abs(g - exact)
        assert np.all(err <= bound), f"fp32 append: max err/bound = {np.max(err / bound):.3g}"
        return dict(mismatch=int(np.sum(g != oracle.round_to_dtype(exact, 'f32'))), n=g.size)
    lo = oracle.round_bf16(exact - bound)
    hi = oracle.round_bf16(exact + bound)
    bad = (g < lo) | (g > hi)
    assert not np.any(bad), (f"bf16 append: {int(bad.sum())} values outside the fp32-accumulation interval, "
                             f"e.g. gpu {g[bad][:4]} exact {exact[bad][:4]} bound {bound[bad][:4]}")
    return dict(mismatch=int(np.sum(g != oracle.round_bf16(exact))), n=g.size)
