"""Host logic of the calibration helpers: the per-layer choice of d."""
import math

import numpy as np
import pytest

from sparse_decode_attention_loki_b200.calibration import choose_d


def test_geometric_spectrum_closed_form():
    # lambda_i = 2^-i: the first d hold (1 - 2^-d) / (1 - 2^-D) of the sum
    lam = [2.0 ** -i for i in range(64)]
    for energy, d in [(0.5, 1), (0.75, 2), (0.9, 4), (0.99, 7), (0.999, 10)]:
        assert choose_d(lam, energy, multiple=1) == d
        assert choose_d(lam, energy, multiple=8) == 8 * math.ceil(d / 8)


def test_flat_spectrum_closed_form():
    lam = [3.0] * 128
    for energy in [0.1, 0.25, 0.5, 0.8, 1.0]:
        assert choose_d(lam, energy, multiple=1) == math.ceil(energy * 128)
        assert choose_d(lam, energy, multiple=16) == min(128, 16 * math.ceil(math.ceil(energy * 128) / 16))


def test_edges():
    lam = [5.0, 1.0, 0.0, 0.0]
    assert choose_d(lam, 1.0, multiple=1) == 2       # the zero tail is never needed
    assert choose_d(lam, 1.0, multiple=8) == 4       # capped at D
    assert choose_d([0.0] * 16, 0.9, multiple=8) == 8
    assert choose_d([1.0, -1e-18], 1.0, multiple=1) == 1   # a negative rounding residue counts as zero
    for bad in [0.0, -0.1, 1.5]:
        with pytest.raises(ValueError):
            choose_d(lam, bad)
    with pytest.raises(ValueError):
        choose_d([1.0, 2.0], 0.5)
    with pytest.raises(ValueError):
        choose_d([], 0.5)
    with pytest.raises(ValueError):
        choose_d(lam, 0.5, multiple=0)


def test_layers_with_steeper_spectra_get_smaller_d():
    D = 128
    ds = [choose_d(list(np.arange(1, D + 1, dtype=float) ** -alpha), 0.9) for alpha in (0.5, 1.0, 1.5, 2.0)]
    assert ds == sorted(ds, reverse=True) and ds[0] > ds[-1]
