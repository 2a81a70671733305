"""GPU PCA calibration (loki_pca_calibrate) against the fp64 oracle.

The oracle's pca_basis is the plain definition (centred covariance, a library
symmetric eigensolver, descending order, largest-magnitude entry positive).
Both sides see the same fp32 (or bf16) keys widened exactly to fp64.  An
eigenvector is determined to about eps * ||C|| / gap, gap = the distance of its
eigenvalue to the nearest other one, so each column is compared within
1e-6 (the fp32 rounding of P) plus that bound.
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import get_workload
from workloads import generators as gen

pytestmark = pytest.mark.gpu


def _gpu_pca(keys_np, dtype=torch.float32):
    import sparse_decode_attention_loki_b200 as L
    k = torch.as_tensor(np.ascontiguousarray(keys_np), dtype=torch.float32).to(dtype).cuda()
    P, w = L.loki_pca_calibrate(k)
    torch.cuda.synchronize()
    return P.cpu().numpy().astype(np.float64), w.cpu().numpy(), k.float().cpu().numpy().astype(np.float64)


def _compare_head(X, P_gpu, w_gpu):
    """X: the exact fp64 keys of one head; P_gpu, w_gpu: the GPU result."""
    P_or, w_or = oracle.pca_basis(X)
    D = X.shape[1]
    scale = max(abs(w_or[0]), 1e-300)
    np.testing.assert_allclose(w_gpu, w_or, rtol=0, atol=1e-12 * scale + 1e-300)
    gaps = np.full(D, np.inf)
    if D > 1:
        d = np.abs(np.diff(w_or))
        gaps[:-1] = np.minimum(gaps[:-1], d)
        gaps[1:] = np.minimum(gaps[1:], d)
    for j in range(D):
        tol = 1e-6 + (1e-12 * scale / gaps[j] if gaps[j] > 0 else np.inf)
        if not np.isfinite(tol):
            continue  # an exactly repeated eigenvalue: only the span is defined
        err = np.abs(P_gpu[:, j] - P_or[:, j]).max()
        if err > tol:
            # the sign rule can differ only if the two largest magnitudes tie
            a = np.sort(np.abs(P_or[:, j]))[::-1]
            assert a[0] - a[1] < 1e-9 and np.abs(P_gpu[:, j] + P_or[:, j]).max() <= tol, (j, err, tol)
    # whatever the spectrum: orthonormal columns and C P = P diag(w)
    C = np.cov(X.T, bias=True)
    np.testing.assert_allclose(P_gpu.T @ P_gpu, np.eye(D), atol=5e-6)
    resid = np.abs(C @ P_gpu - P_gpu * w_gpu[None, :]).max()
    assert resid <= 5e-6 * scale + 1e-12, resid


@pytest.mark.parametrize("name", ["tiny-fp32", "llama2-7b-decode", "llama3-8b-gqa-decode"])
def test_workload_calibration_matches_oracle(name):
    w = get_workload(name)
    heads = min(w.n_kv_heads, 4)
    keys = np.stack([gen.calibration_keys(w, g) for g in range(heads)]).astype(np.float32)
    P, ev, X = _gpu_pca(keys)
    for g in range(heads):
        _compare_head(X[g], P[g], ev[g])


@pytest.mark.parametrize("D,N,H", [(64, 1000, 3), (128, 300, 2), (128, 40, 1), (64, 64, 2)])
def test_random_keys_matches_oracle(D, N, H):
    rng = np.random.default_rng(D * 1000 + N)
    A = rng.standard_normal((H, D, D)) * (0.9 ** np.arange(D))[None, None, :]
    keys = (np.einsum("hnd,hde->hne", rng.standard_normal((H, N, D)), A) + rng.standard_normal((H, 1, D))).astype(
        np.float32)
    P, ev, X = _gpu_pca(keys)
    for g in range(H):
        _compare_head(X[g], P[g], ev[g])


def test_bf16_keys():
    rng = np.random.default_rng(7)
    keys = (rng.standard_normal((2, 500, 128)) * np.linspace(3, 0.1, 128)[None, None, :]).astype(np.float32)
    P, ev, X = _gpu_pca(keys, torch.bfloat16)
    for g in range(2):
        _compare_head(X[g], P[g], ev[g])


def test_single_key_gives_identity():
    """N = 1: the covariance is zero, every eigenvalue 0, no rotation is
    applied and the basis is the identity (ties in index order)."""
    keys = np.random.default_rng(1).standard_normal((2, 1, 64)).astype(np.float32)
    P, ev, _ = _gpu_pca(keys)
    assert np.array_equal(ev, np.zeros_like(ev))
    for g in range(2):
        assert np.array_equal(P[g], np.eye(64))


def test_diagonal_covariance_gives_exact_permutation():
    """Keys +-a_i e_i: the covariance is diagonal with distinct entries, so no
    rotation is needed and P is exactly the permutation that sorts a_i^2
    descending (all signs positive)."""
    D = 128
    rng = np.random.default_rng(3)
    a = rng.permutation(np.arange(1, D + 1)).astype(np.float32) / 8
    X = np.zeros((2 * D, D), dtype=np.float32)
    for i in range(D):
        X[2 * i, i] = a[i]
        X[2 * i + 1, i] = -a[i]
    P, ev, _ = _gpu_pca(X[None])
    order = np.argsort(-a.astype(np.float64), kind="stable")
    expect = np.zeros((D, D))
    expect[order, np.arange(D)] = 1.0
    assert np.array_equal(P[0], expect)
    np.testing.assert_allclose(ev[0], (a.astype(np.float64)[order] ** 2) / D, rtol=1e-15)
