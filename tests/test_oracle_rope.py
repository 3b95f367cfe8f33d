"""Pins for the oracle's 3-D RoPE (CPU only).

Each test holds the oracle to something other than itself: a library rotary
implementation (GPT-J's interleaved rotary in ``transformers``), or a property
the mathematics fixes (orthogonality, relative-position invariance, group
composition, the period of each frequency)."""
import math

import numpy as np
import pytest
import torch

import oracle

SPLITS = [(16, 24, 24), (32, 48, 48), (2, 2, 2)]


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("split", [(16, 24, 24), (32, 48, 48)])
@pytest.mark.parametrize("axis", [0, 1, 2])
def test_single_axis_matches_gptj_rotary(split, axis):
    """With only one axis non-zero, that axis' sub-block must turn exactly as
    GPT-J's interleaved rotary of width d_a (fp32 tables) and the other
    sub-blocks must not move."""
    from transformers.models.gptj import modeling_gptj as gptj
    D = sum(split)
    n = 40
    x = _rand((n, D), 1)
    pos = np.zeros((n, 3))
    pos[:, axis] = np.arange(n)
    y = oracle.rope3d(x, pos, split)
    lo = sum(split[:axis])
    da = split[axis]
    table = gptj.create_sinusoidal_positions(n, da)             # [n, da] = sin | cos
    sin, cos = torch.split(table, da // 2, dim=-1)
    xt = torch.tensor(x[:, lo:lo + da], dtype=torch.float32)[None, :, None, :]
    ref = gptj.apply_rotary_pos_emb(xt, sin[None], cos[None])[0, :, 0, :].double().numpy()
    np.testing.assert_allclose(y[:, lo:lo + da], ref, atol=2e-5, rtol=0)
    mask = np.ones(D, bool)
    mask[lo:lo + da] = False
    assert np.array_equal(y[:, mask], x[:, mask])


@pytest.mark.parametrize("split", SPLITS)
def test_zero_position_is_identity(split):
    x = _rand((17, sum(split)), 2)
    y = oracle.rope3d(x, np.zeros((17, 3)), split)
    assert np.array_equal(x, y)


@pytest.mark.parametrize("split", SPLITS)
def test_pair_norms_preserved(split):
    D = sum(split)
    x = _rand((64, D), 3)
    pos = np.random.default_rng(4).uniform(-40, 40, (64, 3))
    y = oracle.rope3d(x, pos, split)
    nx = np.hypot(x[:, 0::2], x[:, 1::2])
    ny = np.hypot(y[:, 0::2], y[:, 1::2])
    np.testing.assert_allclose(ny, nx, rtol=1e-14, atol=0)


@pytest.mark.parametrize("split", SPLITS)
def test_relative_position_invariance(split):
    """(R(p+d) q) . (R(p'+d) k) == (R(p) q) . (R(p') k), fractional d on every
    axis (the stream-clock shift invariance)."""
    D = sum(split)
    rng = np.random.default_rng(5)
    q, k = rng.standard_normal((32, D)), rng.standard_normal((32, D))
    p, pp = rng.uniform(-30, 30, (32, 3)), rng.uniform(-30, 30, (32, 3))
    for delta in ([0.15, 0.0, 0.0], [7.0, -3.5, 11.25], [-1000.0, 0.0, 0.0]):
        d = np.asarray(delta)[None]
        a = np.sum(oracle.rope3d(q, p + d, split) * oracle.rope3d(k, pp + d, split), axis=1)
        b = np.sum(oracle.rope3d(q, p, split) * oracle.rope3d(k, pp, split), axis=1)
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-9 * max(1.0, abs(delta[0]) / 10))


@pytest.mark.parametrize("split", SPLITS)
def test_composition(split):
    D = sum(split)
    rng = np.random.default_rng(6)
    x = rng.standard_normal((16, D))
    p1, p2 = rng.uniform(-9, 9, (16, 3)), rng.uniform(-9, 9, (16, 3))
    a = oracle.rope3d(oracle.rope3d(x, p2, split), p1, split)
    b = oracle.rope3d(x, p1 + p2, split)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_frequency_period_per_pair():
    """Pair j of axis a returns to itself after a turn of 2*pi / theta_j with
    theta_j = 10000^(-2j/d_a): pins the exponent and the pair index."""
    split = (16, 24, 24)
    D = sum(split)
    x = _rand((1, D), 7)
    lo = 0
    for a, da in enumerate(split):
        for j in range(da // 2):
            period = 2 * math.pi * 10000.0 ** (2 * j / da)
            pos = np.zeros((1, 3))
            pos[0, a] = period
            y = oracle.rope3d(x, pos, split)
            sl = slice(lo + 2 * j, lo + 2 * j + 2)
            np.testing.assert_allclose(y[0, sl], x[0, sl], atol=1e-8 * max(1.0, period / 100))
            # a quarter period turns (x0, x1) into (-x1, x0): pins the direction
            pos[0, a] = period / 4
            y = oracle.rope3d(x, pos, split)
            np.testing.assert_allclose(y[0, sl], [-x[0, lo + 2 * j + 1], x[0, lo + 2 * j]], atol=1e-8 * max(1.0, period / 100))
        lo += da


def test_multi_head_broadcast():
    split = (16, 24, 24)
    x = _rand((5, 3, 64), 8)
    pos = np.random.default_rng(9).uniform(-5, 5, (5, 3))
    y = oracle.rope3d(x, pos, split)
    for h in range(3):
        np.testing.assert_array_equal(y[:, h], oracle.rope3d(np.ascontiguousarray(x[:, h]), pos, split))
