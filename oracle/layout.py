"""Window layout and (t, h, w) positions -- the oracle's own reading.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Sources and readings:
  * "StreamRender-H3" (molayo1419.me), streaming context section: each chunk
    is generated in a window holding a sink (the initial scene, kept for the
    whole session) and recent history; the window's position template is
    fixed after the first window.  Reading: window-relative positions with the
    chunk's video frames at t = 0, 1, ... and the context frames just before
    it, chronologically, at t = -n_ctx .. -1 (the sink earliest).
  * "AlayaRenderer-Flash" (aitrends.kr), technical details: three tiers of
    history, recent at full resolution, older progressively pooled; the first
    generated frame stays as the global appearance anchor.  Reading: a pooled
    cell sits at (t of its frame, mean row, mean col) of its members.
  * "MiniMax-H3 deep dive" (fiv.co.kr), audio VAE row: audio latents at 40 Hz;
    24 fps video / 4 = 6 latent frames per second.  Reading: audio token i sits
    at t = i * 6 / 40 latent frames, h = w = 0.
  * Persistent prompt KV ("AlayaRenderer-Flash", key contributions): reading:
    not rotated (position (0, 0, 0)).

Segment order in the attention buffer (each segment's capacity is its
valid length rounded up to a multiple of 128):
    prompt, sink, tiers oldest -> newest, recent, chunk.
Inside a segment tokens are frame-major then row-major (h, then w); in the
chunk the audio tokens follow the video tokens.
"""
from __future__ import annotations

from typing import List, Tuple

TILE = 128


def frame_token_rc(i: int, grid_w: int) -> Tuple[int, int]:
    """(row, col) of token i of a frame (row-major)."""
    return i // grid_w, i % grid_w


def chunk_positions(spec) -> List[Tuple[float, float, float]]:
    out = []
    for f, n in enumerate(spec.chunk_frame_tokens()):
        for i in range(n):
            r, c = frame_token_rc(i, spec.grid_w)
            out.append((float(f), float(r), float(c)))
    for i in range(spec.chunk_audio_tokens):
        out.append((i * spec.latent_fps / spec.audio_rate, 0.0, 0.0))
    return out


def context_plan(spec):
    """Context frames oldest first as (t, role, pool_h, pool_w, n_tokens);
    role is 'sink', 'tier<k>' (k = 0 is the oldest tier) or 'recent'."""
    n_tok = spec.context_frame_tokens()
    n_frames = len(n_tok)
    roles = []
    f = 0
    for _ in range(min(spec.sink_frames, n_frames)):
        roles.append(("sink", 1, 1))
        f += 1
    for k, (nf, ph, pw) in enumerate(spec.tiers):
        for _ in range(nf):
            assert f < n_frames, "more tier frames than context frames"
            roles.append((f"tier{k}", ph, pw))
            f += 1
    while f < n_frames:
        roles.append(("recent", 1, 1))
        f += 1
    return [(float(i - n_frames), roles[i][0], roles[i][1], roles[i][2], n_tok[i])
            for i in range(n_frames)]


def pooled_cells(grid_h: int, grid_w: int, ph: int, pw: int):
    """Cells of a ph x pw ceil-mode pooling, row-major: (r0, r1, c0, c1, mean_row, mean_col)."""
    out = []
    for r in range(-(-grid_h // ph)):
        for c in range(-(-grid_w // pw)):
            r0, r1 = r * ph, min((r + 1) * ph, grid_h)
            c0, c1 = c * pw, min((c + 1) * pw, grid_w)
            rows = list(range(r0, r1))
            cols = list(range(c0, c1))
            out.append((r0, r1, c0, c1, sum(rows) / len(rows), sum(cols) / len(cols)))
    return out


def segment_names(spec) -> List[str]:
    names = ["prompt"]
    if spec.sink_frames and spec.context_video_tokens:
        names.append("sink")
    names += [f"tier{k}" for k in range(len(spec.tiers))]
    plan = context_plan(spec)
    if any(role == "recent" for _, role, _, _, _ in plan):
        names.append("recent")
    names.append("chunk")
    return names


def segment_lengths(spec) -> List[int]:
    """Valid token count per segment, in segment order."""
    plan = context_plan(spec)
    lens = {"prompt": spec.prompt_len, "chunk": spec.chunk_len}
    for t, role, ph, pw, n in plan:
        if role.startswith("tier"):
            assert n == spec.frame_tokens, "pooled frames must be complete"
            cells = len(pooled_cells(spec.grid_h, spec.grid_w, ph, pw))
            lens[role] = lens.get(role, 0) + cells
        else:
            lens[role] = lens.get(role, 0) + n
    return [lens.get(name, 0) for name in segment_names(spec)]


def capacities(specs) -> List[int]:
    """Per-segment capacity shared by a batch of sessions with the same
    segment names: the largest valid length rounded up to 128."""
    names = segment_names(specs[0])
    caps = []
    for si in range(len(names)):
        m = 0
        for sp in specs:
            assert segment_names(sp) == names
            m = max(m, segment_lengths(sp)[si])
        caps.append(max(TILE, -(-m // TILE) * TILE))
    return caps


def segment_offsets(caps: List[int]) -> List[int]:
    out, acc = [], 0
    for c in caps:
        out.append(acc)
        acc += c
    return out
