"""Shifted-window attention with ring-buffer KV, as in a causal streaming VAE
decoder.

Source: "StreamRender-H3" (molayo1419.me), causal VAE section:
  * each call decodes 2 latent frames; every layer attends only to the KV of
    the 2 current and the 4 previous latent frames, never to future frames;
  * non-overlapping 16x16 token windows, shifted by half a window every
    other layer to exchange information between neighbours;
  * each window's KV lives in a preallocated ring buffer; position encoding
    and the cache write happen once; window partition and merge are index
    gathers; empty cache slots are hidden by per-slot valid lengths instead
    of a mask.

Readings: inside a call the two current frames see each other (causality at
the granularity of a call); RoPE on (t, h, w) with t the absolute latent
frame index, applied once when a frame enters the ring (attention only sees
position differences); a window's tokens are packed valid-first (attention is
invariant to key order), so partial windows at the grid edge are ragged
segments.

Everything runs in the library's kernels: sr_gather_tokens (V into the
ring), sr_gather_rope3d_tokens (K into the ring and the queries into their
windows, rotated on the way), sr_chunk_attention_fwd (attention: batch =
windows, segments = ring slots) and sr_scatter_tokens (merge).
"""
from __future__ import annotations

import math
from typing import List, Sequence

import numpy as np
import torch

from . import capi
from .window import _mark


class WindowPartition:
    """Windows of `window` x `window` tokens tiling a gh x gw grid whose origin
    is moved by -shift (shift = window / 2 on alternate layers)."""

    def __init__(self, gh: int, gw: int, window: int = 16, shift: int = 0):
        self.gh, self.gw, self.window, self.shift = gh, gw, window, shift
        self.tokens: List[List[int]] = []   # row-major token indices of each window (valid only)
        for r0 in range(-shift, gh, window):
            for c0 in range(-shift, gw, window):
                rows = range(max(r0, 0), min(r0 + window, gh))
                cols = range(max(c0, 0), min(c0 + window, gw))
                toks = [r * gw + c for r in rows for c in cols]
                if toks:
                    self.tokens.append(toks)
        self.n_windows = len(self.tokens)
        self.counts = np.array([len(t) for t in self.tokens], dtype=np.int32)

    def frame_index(self, frames: int) -> np.ndarray:
        """[n_windows][frames * window^2] int32: the windows' tokens of `frames`
        consecutive frames packed valid-first (frame f's tokens offset by
        f * gh * gw), padded with -1."""
        slots = frames * self.window * self.window
        out = np.full((self.n_windows, slots), -1, dtype=np.int32)
        per = self.gh * self.gw
        for w, toks in enumerate(self.tokens):
            idx = [f * per + t for f in range(frames) for t in toks]
            out[w, :len(idx)] = idx
        return out


class RingWindowAttention:
    """One layer's windowed attention with a per-window KV ring of
    (current + history) latent frames."""

    def __init__(self, grid_hw, n_heads: int, head_dim: int, rope_split, shift: int = 0, window: int = 16,
                 frames_per_call: int = 2, history_frames: int = 4, rope_base: float = 10000.0, device="cuda"):
        self.part = WindowPartition(grid_hw[0], grid_hw[1], window, shift)
        self.H, self.D = n_heads, head_dim
        self.split, self.base = tuple(rope_split), rope_base
        self.fpc, self.slots = frames_per_call, frames_per_call + history_frames
        self.slot_cap = window * window
        self.device = torch.device(device)
        W, H, D, S = self.part.n_windows, n_heads, head_dim, self.slot_cap
        kw = dict(device=self.device)
        self.k_ring = torch.zeros(W, H, self.slots * S, D, dtype=torch.bfloat16, **kw)
        self.v_ring = torch.zeros(W, H, self.slots * S, D, dtype=torch.bfloat16, **kw)
        self.q_cap = self.fpc * S
        self.q_att = torch.zeros(W, H, self.q_cap, D, dtype=torch.bfloat16, **kw)
        self.o_win = torch.zeros(W, self.q_cap, H, D, dtype=torch.bfloat16, **kw)
        self.lse = torch.zeros(W, H, self.q_cap, dtype=torch.float32, **kw)
        self.status = torch.zeros(1, dtype=torch.int32, **kw)
        self.idx_q = torch.from_numpy(self.part.frame_index(self.fpc)).to(self.device)
        per = self.part.gh * self.part.gw
        one = self.part.frame_index(1)
        self.idx_kv = [torch.from_numpy(np.where(one >= 0, one + f * per, -1).astype(np.int32)).to(self.device)
                       for f in range(self.fpc)]
        self.q_len = torch.from_numpy(self.fpc * self.part.counts).to(self.device)
        # valid length of every ring slot after call c: slots written so far hold a window's count
        self.kv_len_phase = []
        for c in range(self.slots // self.fpc):
            lens = np.zeros((W, self.slots), dtype=np.int32)
            lens[:, :min(self.slots, (c + 1) * self.fpc)] = self.part.counts[:, None]
            self.kv_len_phase.append(torch.from_numpy(lens).to(self.device))
        ws = capi.sr_chunk_attention_workspace_bytes(W, H, D, self.q_cap)
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, **kw) if ws else None
        # positions of the current frames: the fixed table (f, row, col) plus
        # the call's first frame index t0 on the t axis, which the rotating
        # kernels add themselves from a device clock (fp64): a call never waits
        # for the host and a replayed graph sees the new t0.  The clock is
        # advanced by frames_per_call at the start of every call's prepare, so
        # consecutive calls need no host write; a jump in t0 sets it directly.
        self.pos_base = self.frame_positions(0)
        self.t0_dev = torch.zeros(1, dtype=torch.float64, **kw)
        self.t0_next = None   # t0 the device clock reaches at the next advance
        self.calls = 0
        self.graphs = {}

    def frame_positions(self, t0: int) -> torch.Tensor:
        """(t, h, w) of the current frames' tokens, t absolute."""
        gh, gw = self.part.gh, self.part.gw
        r, c = np.divmod(np.arange(gh * gw), gw)
        pos = [np.stack([np.full(gh * gw, t0 + f), r, c], axis=1) for f in range(self.fpc)]
        return torch.from_numpy(np.concatenate(pos).astype(np.float32)).to(self.device)

    def _state(self):
        """(first ring slot of this call, valid-length phase) from the call count."""
        return (self.calls * self.fpc) % self.slots, min(self.calls, len(self.kv_len_phase) - 1)

    def _prepare(self, q, k, v, slot0: int, stream=None) -> None:
        """Positions, then the cache write of the current frames (V copied, K
        rotated on the way into its ring slot) and the partition of the
        queries (rotated on the way): one gather launch each."""
        S = self.slot_cap
        capi.sr_stream_clock_advance(self.t0_dev, float(self.fpc), stream=stream)
        for f in range(self.fpc):
            sl = (slot0 + f) % self.slots
            ring_k = self.k_ring[:, :, sl * S:(sl + 1) * S].permute(0, 2, 1, 3)
            ring_v = self.v_ring[:, :, sl * S:(sl + 1) * S].permute(0, 2, 1, 3)
            capi.sr_gather_tokens(ring_v, v, self.idx_kv[f], stream=stream)
            capi.sr_gather_rope3d_tokens(ring_k, k, self.idx_kv[f], self.pos_base, self.split, self.base,
                                         t_origin=self.t0_dev, stream=stream)
        capi.sr_gather_rope3d_tokens(self.q_att.permute(0, 2, 1, 3), q, self.idx_q, self.pos_base, self.split,
                                     self.base, t_origin=self.t0_dev, stream=stream)

    def _set_t0(self, t0: int) -> None:
        """Make the next advance of the device clock land on t0: nothing to do
        for consecutive calls; otherwise one host-to-device copy (in stream
        order, no kernel)."""
        if self.t0_next != t0:
            self.t0_dev.copy_(torch.tensor([float(t0 - self.fpc)], dtype=torch.float64))
        self.t0_next = t0 + self.fpc

    def _attend(self, phase: int, stream=None) -> None:
        S = self.slot_cap
        capi.sr_chunk_attention_fwd(self.q_att, self.k_ring, self.v_ring, self.o_win, self.lse,
                                    [S] * self.slots, self.kv_len_phase[phase], self.q_len,
                                    1.0 / math.sqrt(self.D), self.status, workspace=self.workspace, stream=stream)

    def _merge(self, out, stream=None) -> None:
        capi.sr_scatter_tokens(out, self.o_win, self.idx_q, stream=stream)

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, t0: int,
                 out: torch.Tensor = None, stream=None, marks=None) -> torch.Tensor:
        """q, k, v: the current frames' tokens [frames_per_call * gh * gw, H, D]
        (token-major, before RoPE); t0: absolute latent index of the first
        current frame.  Returns o of the same shape.  `marks`: optional pair
        of CUDA events recorded around the attention launch."""
        n_tok = self.fpc * self.part.gh * self.part.gw
        assert q.shape == (n_tok, self.H, self.D) and k.shape == q.shape and v.shape == q.shape
        if out is None:
            out = torch.zeros_like(q)
        slot0, phase = self._state()
        self._set_t0(t0)
        self._prepare(q, k, v, slot0, stream)
        _mark(marks, 0, stream)
        self._attend(phase, stream)
        _mark(marks, 1, stream)
        self._merge(out, stream)
        self.calls += 1
        return out

    def graphed(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, t0: int, out: torch.Tensor,
                marks=None) -> torch.Tensor:
        """The same call replayed from CUDA graphs (no per-launch host work).

        q, k, v and out must be the same tensors (addresses) on every call.
        Each ring state (first slot, valid-length phase) -- five in all for
        the default 2 + 4 frames -- is captured the first time it occurs,
        after that call has run eagerly; a call then costs three graph launches
        (prepare, attention, merge) on the current stream, with `marks`
        recorded around the attention graph."""
        slot0, phase = self._state()
        key = (slot0, phase)
        if key not in self.graphs:
            self(q, k, v, t0, out=out, marks=marks)
            torch.cuda.synchronize()
            gs = [torch.cuda.CUDAGraph() for _ in range(3)]
            with torch.cuda.graph(gs[0]):
                self._prepare(q, k, v, slot0)
            with torch.cuda.graph(gs[1]):
                self._attend(phase)
            with torch.cuda.graph(gs[2]):
                self._merge(out)
            self.graphs[key] = gs
            return out
        gs = self.graphs[key]
        self._set_t0(t0)
        gs[0].replay()
        _mark(marks, 0, None)
        gs[1].replay()
        _mark(marks, 1, None)
        gs[2].replay()
        self.calls += 1
        return out
