"""Seeded synthetic inputs for the chunk-streaming joint attention step.

This module holds shapes and random draws only: no RoPE, pooling, layout or
attention arithmetic lives here.  It is the one module that both the fp64
oracle (``oracle/``) and the CUDA path's tests and bench import, so that both
sides consume the same bf16 bytes.

Workload shapes follow the pages:
  * latent geometry: the visual VAE compresses 16x in space and 4x in time and
    the DiT patchifies (1,2,2), so a 1344x768 frame is a 24x42 (rows x cols)
    token grid, 1,008 tokens per latent frame; audio latents run at 40 Hz and
    24 fps video gives 6 latent frames per second ("MiniMax-H3 deep dive",
    fiv.co.kr: H3-VisualVAE / H3-AudioVAE table and the transformer config
    table);
  * the streaming window: a sink (initial scene) kept for the whole session
    plus recent outputs as context ("StreamRender-H3", molayo1419.me: section
    on streaming context), older history pooled into coarser tiers and a
    persistent style-prompt KV in every self-attention ("AlayaRenderer-Flash",
    aitrends.kr: key contributions and technical details).

Draw order for one session (fixed; each draw is ``standard_normal`` in fp32,
times ``value_scale``, rounded to nearest-even bf16, token-major [L, H, D]):
  prompt K, prompt V; for every context frame in chronological order (the sink
  first, then history oldest to newest, all at full resolution): K, V; then the
  chunk Q, K, V (video tokens first, audio tokens after).
The ragged batch draws its three length factors from ``default_rng(1000+s)``
before drawing session ``s`` from ``default_rng(s)``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Tuple

import numpy as np
import torch

GRID_H_FULL = 24          # 768 / 16 / 2
GRID_W_FULL = 42          # 1344 / 16 / 2
LATENT_FPS = 6.0          # 24 fps / 4 (temporal compression)
AUDIO_RATE = 40.0         # audio latent tokens per second


@dataclasses.dataclass(frozen=True)
class SessionSpec:
    """Shape of one streaming session (one layer, all heads)."""
    name: str
    n_heads: int
    head_dim: int
    rope_split: Tuple[int, int, int]      # (d_t, d_h, d_w)
    rope_base: float
    grid_h: int                           # token rows per latent frame
    grid_w: int                           # token cols per latent frame
    prompt_len: int
    context_video_tokens: int             # full-resolution context tokens (sink + history)
    sink_frames: int                      # oldest context frames kept at full resolution as the sink
    tiers: Tuple[Tuple[int, int, int], ...]  # (n_frames, pool_h, pool_w), oldest tier first
    chunk_video_tokens: int
    chunk_audio_tokens: int
    value_scale: float
    latent_fps: float = LATENT_FPS
    audio_rate: float = AUDIO_RATE

    @property
    def frame_tokens(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def context_frames(self) -> int:
        return -(-self.context_video_tokens // self.frame_tokens)

    @property
    def chunk_len(self) -> int:
        return self.chunk_video_tokens + self.chunk_audio_tokens

    def context_frame_tokens(self) -> List[int]:
        """Token count of each context frame, oldest first (last may be partial)."""
        out, left = [], self.context_video_tokens
        while left > 0:
            n = min(left, self.frame_tokens)
            out.append(n)
            left -= n
        return out

    def chunk_frame_tokens(self) -> List[int]:
        out, left = [], self.chunk_video_tokens
        while left > 0:
            n = min(left, self.frame_tokens)
            out.append(n)
            left -= n
        return out


def _spec(name, H, D, split, Gh, Gw, Lp, ctx_tokens, sink, tiers, chunk_video, chunk_audio, scale):
    return SessionSpec(name=name, n_heads=H, head_dim=D, rope_split=split, rope_base=10000.0,
                       grid_h=Gh, grid_w=Gw, prompt_len=Lp, context_video_tokens=ctx_tokens,
                       sink_frames=sink, tiers=tuple(tiers), chunk_video_tokens=chunk_video,
                       chunk_audio_tokens=chunk_audio, value_scale=scale)


FT = GRID_H_FULL * GRID_W_FULL
INV_SQRT2 = 1.0 / math.sqrt(2.0)

# tiny CPU-checkable case: 1 head x 64, grid 6x8, 2 chunk frames + 4 audio,
# 2 context frames, 16 prompt tokens, N(0,1)
TINY = _spec("tiny", 1, 64, (16, 24, 24), 6, 8, 16, 2 * 48, 1, (), 2 * 48, 4, 1.0)
# one streaming chunk at 1344x768: 3 frames + 20 audio, sink + 3 recent, 256 prompt
CHUNK = _spec("chunk", 40, 128, (32, 48, 48), GRID_H_FULL, GRID_W_FULL, 256, 4 * FT, 1, (),
              3 * FT, 20, INV_SQRT2)
# the same chunk with 3-tier history: sink + 12 frames pooled 4x4 + 9 pooled 2x2 + 3 full
CHUNK_TIERED = _spec("chunk_tiered", 40, 128, (32, 48, 48), GRID_H_FULL, GRID_W_FULL, 256,
                     25 * FT, 1, ((12, 4, 4), (9, 2, 2)), 3 * FT, 20, 1.0)
# full 5 s clip, non-streaming: 30 frames + 200 audio, 256 prompt, no context
CLIP = _spec("clip", 40, 128, (32, 48, 48), GRID_H_FULL, GRID_W_FULL, 256, 0, 0, (),
             30 * FT, 200, INV_SQRT2)

CONFIGS: Dict[int, SessionSpec] = {1: TINY, 2: CHUNK, 3: CHUNK_TIERED, 4: CLIP}
RAGGED_SESSIONS = 20


def ragged_spec(s: int) -> SessionSpec:
    """Session ``s`` (1-based) of the ragged batch: a one-chunk session with
    prompt, context and chunk-video lengths scaled by factors in [0.9, 1.1]."""
    f = np.random.default_rng(1000 + s).uniform(0.9, 1.1, size=3)
    lp = int(round(256 * float(f[0])))
    lc = int(round(4 * FT * float(f[1])))
    lk = int(round(3 * FT * float(f[2])))
    return _spec(f"ragged_{s}", 40, 128, (32, 48, 48), GRID_H_FULL, GRID_W_FULL, lp, lc, 1, (),
                 lk, 20, INV_SQRT2)


def ragged_batch() -> List[Tuple[SessionSpec, int]]:
    return [(ragged_spec(s), s) for s in range(1, RAGGED_SESSIONS + 1)]


def session_list(config: int) -> List[Tuple[SessionSpec, int]]:
    """(spec, seed) pairs for a config number 1..5."""
    if config == 5:
        return ragged_batch()
    return [(CONFIGS[config], 0)]


def scaled(spec: SessionSpec, **kw) -> SessionSpec:
    """A copy of ``spec`` with some fields replaced (smaller parity cases)."""
    return dataclasses.replace(spec, **kw)


def _draw(rng: np.random.Generator, n: int, spec: SessionSpec) -> torch.Tensor:
    x = rng.standard_normal((n, spec.n_heads, spec.head_dim), dtype=np.float32)
    if spec.value_scale != 1.0:
        x = x * np.float32(spec.value_scale)
    return torch.from_numpy(x).to(torch.bfloat16)


@dataclasses.dataclass
class SessionInputs:
    """bf16 CPU tensors, token-major [L, H, D]."""
    prompt_k: torch.Tensor
    prompt_v: torch.Tensor
    ctx_k: List[torch.Tensor]      # one per context frame, oldest first, full resolution
    ctx_v: List[torch.Tensor]
    q: torch.Tensor                # chunk: video tokens then audio tokens
    k: torch.Tensor
    v: torch.Tensor


def draw_session(spec: SessionSpec, seed: int) -> SessionInputs:
    rng = np.random.default_rng(seed)
    pk = _draw(rng, spec.prompt_len, spec)
    pv = _draw(rng, spec.prompt_len, spec)
    ck, cv = [], []
    for n in spec.context_frame_tokens():
        ck.append(_draw(rng, n, spec))
        cv.append(_draw(rng, n, spec))
    q = _draw(rng, spec.chunk_len, spec)
    k = _draw(rng, spec.chunk_len, spec)
    v = _draw(rng, spec.chunk_len, spec)
    return SessionInputs(pk, pv, ck, cv, q, k, v)


def draw_tensor(shape, seed: int, scale: float = 1.0) -> torch.Tensor:
    """A standalone seeded bf16 tensor (kernel-level parity cases)."""
    x = np.random.default_rng(seed).standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        x = x * np.float32(scale)
    return torch.from_numpy(x).to(torch.bfloat16)


def draw_positions(n: int, seed: int, spread: float = 32.0) -> torch.Tensor:
    """Seeded fp32 (t, h, w) positions, uniform in [-spread, spread)."""
    x = np.random.default_rng(seed).uniform(-spread, spread, size=(n, 3)).astype(np.float32)
    return torch.from_numpy(x)


@dataclasses.dataclass
class MovingInputs:
    """Extra bf16 tensors for the prefix / moving-part split of a window:
    queries of the fixed prefix (prompt then sink tokens) and recomputed
    queries, keys and values of the recent frames (token-major [L, H, D])."""
    prefix_q: torch.Tensor
    recent_q: torch.Tensor
    recent_k: torch.Tensor
    recent_v: torch.Tensor


def recent_tokens(spec: SessionSpec) -> int:
    """Full-resolution context tokens after the sink and the pooled tiers."""
    sizes = spec.context_frame_tokens()
    skip = min(spec.sink_frames, len(sizes)) + sum(n for n, _, _ in spec.tiers)
    return sum(sizes[skip:])


def sink_tokens(spec: SessionSpec) -> int:
    return sum(spec.context_frame_tokens()[:spec.sink_frames])


def draw_moving(spec: SessionSpec, seed: int) -> MovingInputs:
    """Drawn from default_rng([seed, 1]) in this order: prefix Q, recent Q,
    recent K, recent V (same distribution as the session's tensors)."""
    rng = np.random.default_rng([seed, 1])
    n_prefix = spec.prompt_len + sink_tokens(spec)
    n_recent = recent_tokens(spec)
    return MovingInputs(_draw(rng, n_prefix, spec), _draw(rng, n_recent, spec), _draw(rng, n_recent, spec),
                        _draw(rng, n_recent, spec))
