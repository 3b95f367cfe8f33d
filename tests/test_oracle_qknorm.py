"""Pins for the oracle's QK normalisation (CPU only)."""
import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


@pytest.mark.parametrize("D", [64, 128])
def test_matches_torch_rms_norm(D):
    x = _rand((50, 3, D), 1, 3.0)
    g = _rand((D,), 2)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (D,), torch.from_numpy(g), eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.rms_norm(x, g, 1e-6), ref, rtol=0, atol=1e-13)


def test_unit_gain_gives_unit_rms_and_scale_invariance():
    x = _rand((40, 128), 3, 5.0)
    y = oracle.rms_norm(x, np.ones(128), 0.0)
    np.testing.assert_allclose(np.sqrt((y ** 2).mean(axis=1)), 1.0, atol=1e-14)
    np.testing.assert_allclose(oracle.rms_norm(7.5 * x, np.ones(128), 0.0), y, atol=1e-14)


def test_eps_damps_small_vectors():
    x = np.full((1, 64), 1e-4)
    y = oracle.rms_norm(x, np.ones(64), 1e-6)
    # mean(x^2) = 1e-8 << eps: y = x / sqrt(1e-8 + 1e-6)
    np.testing.assert_allclose(y, x / np.sqrt(1e-8 + 1e-6), rtol=1e-14)
