"""Windowed attention of a causal streaming VAE decoder -- fp64 reference.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: "StreamRender-H3" (molayo1419.me), causal VAE section: each call
decodes 2 latent frames; every layer attends only to the 2 current and the
4 previous latent frames; non-overlapping 16x16 token windows, shifted by
half a window every other layer.  Readings: the two current frames see each
other; a token at grid (r, c) belongs to window ((r + shift) // 16,
(c + shift) // 16); RoPE on (t, h, w) with t the absolute frame index.
Written per query token, straight from that definition.
"""
from __future__ import annotations

import numpy as np

from . import attention, rope3d, _f64


def window_of(r: int, c: int, window: int, shift: int):
    return (r + shift) // window, (c + shift) // window


def window_attention_reference(q, k, v, grid_hw, t0: int, call_frames: int, history: int, split,
                               window: int = 16, shift: int = 0, base: float = 10000.0, heads=None):
    """q, k, v: all frames so far [F, gh*gw, H, D] (the last `call_frames`
    frames are the current call, starting at absolute frame t0 + F - call_frames).
    Returns O [call_frames * gh * gw, H', D] for the current frames."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    F, T, H, D = q.shape
    gh, gw = grid_hw
    heads = list(range(H)) if heads is None else list(heads)
    first = F - call_frames
    lo = max(0, first - history)
    out = np.zeros((call_frames * T, len(heads), D))
    # group the tokens of frames [lo, F) by window
    members = {}
    for f in range(lo, F):
        for i in range(T):
            r, c = divmod(i, gw)
            members.setdefault(window_of(r, c, window, shift), []).append((f, i))
    for wid, toks in members.items():
        kf = np.array([f for f, _ in toks])
        ki = np.array([i for _, i in toks])
        pos_k = np.stack([t0 + kf, ki // gw, ki % gw], axis=1).astype(np.float64)
        cur = [(f, i) for f, i in toks if f >= first]
        qf = np.array([f for f, _ in cur])
        qi = np.array([i for _, i in cur])
        pos_q = np.stack([t0 + qf, qi // gw, qi % gw], axis=1).astype(np.float64)
        for hi, h in enumerate(heads):
            kr = rope3d(k[kf, ki, h], pos_k, split, base)
            qr = rope3d(q[qf, qi, h], pos_q, split, base)
            o, _ = attention(qr, kr, v[kf, ki, h], 1.0 / np.sqrt(D))
            out[(qf - first) * T + qi, hi] = o
    return out
