"""Offline PCA calibration of the key basis P, and a per-layer choice of d.

The pages calibrate the PCA transform offline on a calibration set ("Loki:
Low-rank Keys for Efficient Sparse Attention", atlas.scime.ai summary, summary
paragraph).  Calibration is not on the decode path: it runs once, before any
decode step, and hands P to the library as an input.  `pca_bases_gpu` runs
the library's own kernels (loki_pca_calibrate: fp64 covariance and a Jacobi
eigensolver on the device).  The principal directions are ordered by
descending eigenvalue (column j of P = direction j) and the sign of each
column makes its largest-magnitude entry positive.

`choose_d` is a per-layer reduced-dimension policy: the pages vary d across
layers in an ablation and report no clear effect on quality (summary page,
section "Measured effects reported in the paper"); they give no rule, so the
rule here is the plainest one, the fewest leading principal dimensions that
hold a given fraction of the key variance.
"""
from __future__ import annotations

import math
from typing import Sequence

import torch


def pca_bases_gpu(calib: torch.Tensor) -> torch.Tensor:
    """calib: [Hkv, N, D] calibration keys (fp32 or bf16) on a CUDA device ->
    P [Hkv, D, D] fp32 on that device, computed by the library's kernels."""
    from .api import loki_pca_calibrate
    P, _ = loki_pca_calibrate(calib.contiguous())
    return P


def choose_d(eigvals: Sequence[float], energy: float, multiple: int = 8) -> int:
    """Smallest d, a multiple of `multiple` (or D itself), whose leading
    eigenvalues hold at least `energy` of their sum.

    eigvals: the D eigenvalues of one head's key covariance, in descending
    order (negative rounding residues count as zero).  For a layer with several
    KV heads, pass each head's values and take the maximum."""
    if not 0.0 < energy <= 1.0:
        raise ValueError(f"energy {energy} outside (0, 1]")
    if multiple < 1:
        raise ValueError(f"multiple {multiple} must be >= 1")
    lam = [max(0.0, float(x)) for x in eigvals]
    D = len(lam)
    if D == 0:
        raise ValueError("no eigenvalues")
    if any(lam[i] < lam[i + 1] for i in range(D - 1)):
        raise ValueError("eigenvalues must be in descending order")
    total = math.fsum(lam)
    if total == 0.0:
        return min(D, multiple)
    for d in range(1, D + 1):
        if math.fsum(lam[:d]) >= energy * total:
            return min(D, -(-d // multiple) * multiple)
    return D
