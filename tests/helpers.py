"""Comparison helpers shared by the GPU parity tests (no method arithmetic)."""
from __future__ import annotations

import numpy as np
import torch

# Attention output tolerance on bf16 outputs with fp32 accumulation, vs the
# fp64 oracle: max-abs 2e-2, mean-abs 2e-3 (the stated parity bar).
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def bf16_ordered(x: torch.Tensor) -> np.ndarray:
    """Map bf16 values to integers whose difference counts ulps (sign-aware)."""
    b = x.detach().cpu().to(torch.bfloat16).contiguous().view(torch.int16).numpy().astype(np.int32)
    return np.where(b < 0, -(b & 0x7FFF), b)


def ulp_diff_bf16(got: torch.Tensor, ref_f64) -> np.ndarray:
    """|got - round_bf16(ref)| in bf16 ulps (ref is rounded to nearest-even)."""
    ref = torch.as_tensor(np.asarray(ref_f64), dtype=torch.float64).to(torch.bfloat16)
    return np.abs(bf16_ordered(got) - bf16_ordered(ref))


def attn_errors(got, ref) -> tuple:
    g = np.asarray(got.detach().cpu().double().numpy() if hasattr(got, "detach") else got, dtype=np.float64)
    d = np.abs(g - np.asarray(ref, dtype=np.float64))
    return float(d.max()), float(d.mean())


def sample_rows(n: int, k: int, seed: int) -> list:
    """Tile boundaries, the ragged tail and k seeded random rows of [0, n)."""
    fixed = {0, 1, n - 1, n - 2}
    for t in range(128, n, 128):
        fixed |= {t - 1, t}
    rng = np.random.default_rng(seed)
    extra = set(rng.choice(n, size=min(k, n), replace=False).tolist())
    return sorted(r for r in fixed | extra if 0 <= r < n)


def assert_rope_close(got, ref, x):
    """Within one bf16 ulp of the fp64 rotation, except where the rotated
    component nearly cancels: there the fp32 rotation's own error (a few
    2^-24 of the pair's norm) may exceed half an ulp of the tiny result, so
    an absolute 2^-21 * |pair| is allowed.  x: the rotated input."""
    ulps = ulp_diff_bf16(got, ref)
    xd = x.double().numpy() if hasattr(x, "double") else np.asarray(x, dtype=np.float64)
    pair = np.repeat(np.hypot(xd[..., 0::2], xd[..., 1::2]), 2, axis=-1)
    err = np.abs(got.double().numpy() - ref)
    assert np.all((ulps <= 1) | (err <= 2.0 ** -21 * pair))
