"""Offline PCA calibration of the key basis P (host side, once per model).

The pages calibrate the PCA transform offline on a calibration set ("Loki:
Low-rank Keys for Efficient Sparse Attention", atlas.scime.ai summary, summary
paragraph).  This helper is not on the decode path: it runs once, before any
decode step, and hands P to the library as an input.  It uses torch's fp64
symmetric eigensolver on the key covariance and orders the principal
directions by descending eigenvalue (column j of P = direction j), with the
sign of each column fixed so that its largest-magnitude entry is positive.
"""
from __future__ import annotations

import torch


def pca_basis(keys: torch.Tensor) -> torch.Tensor:
    """keys: [N, D] calibration keys of one KV head -> P [D, D] fp32 (CPU)."""
    X = keys.detach().to("cpu", torch.float64)
    Xc = X - X.mean(dim=0, keepdim=True)
    C = Xc.T @ Xc / X.shape[0]
    w, V = torch.linalg.eigh(C)
    order = torch.argsort(w, descending=True, stable=True)
    V = V[:, order]
    lead = V.abs().argmax(dim=0)
    signs = torch.sign(V[lead, torch.arange(V.shape[1])])
    signs[signs == 0] = 1.0
    return (V * signs).to(torch.float32)


def pca_bases(calib) -> torch.Tensor:
    """One basis per KV head: calib is a sequence of [N, D] arrays/tensors ->
    P [Hkv, D, D] fp32 (CPU)."""
    return torch.stack([pca_basis(torch.as_tensor(c)) for c in calib])
