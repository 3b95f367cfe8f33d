"""Streaming window: persistent per-layer KV buffers, their segment layout and
the window position template; the streaming step (KV append, RoPE,
attention), the window slide after a chunk (tier re-pooling over frame
rings), the prefix / moving-part split, CUDA-graph replay of the step and a
host-buffer pipeline.

Sources:
  * "StreamRender-H3" (molayo1419.me), streaming context section: a sink
    (initial scene, kept all session) plus recent history; bidirectional
    attention in the window; the position template of the first window is
    reused afterwards; inference acceleration section: persistent per-layer KV
    buffers in the attention kernel's layout, only the dynamic region updated
    in place, lengths and offsets reused without host-device syncs.
  * "AlayaRenderer-Flash" (aitrends.kr), key contributions and technical
    details: three history tiers (recent full resolution, older pooled), the
    first generated frame kept as the appearance anchor, persistent
    style-prompt KV in every self-attention.
  * "MiniMax-H3 deep dive" (fiv.co.kr): audio latents at 40 Hz, 6 latent
    frames per second, a single token sequence for video and audio.

Readings (the pages leave them open): window-relative positions with the
chunk's frames at t = 0, 1, ... and the context frames at t = -n .. -1 (the
sink earliest); audio token i at t = i * 6 / 40, h = w = 0; pooled cells at
(t, mean member row, mean member col); the prompt at position 0.  q . k after
RoPE depends on position differences only, so every rotation adds a stream
clock (fp64, on the device) to the template t: a slide of n frames advances
the clock by n while the frames' template t fall by n, so a history frame
keeps its rotated keys, rotated once when it enters a ring slot (pooled or
appended, fused into that call).  Only what floats with the chunk is rotated
every step: the chunk's keys (fused into their append), the queries and the
prefix (prompt and sink, whose template places stay fixed relative to the
chunk).  K is also kept pre-RoPE (``k_raw``) where it is pooled later, so
rotation never compounds rounding.  After a chunk its
clean frames become the newest history and every tier hands its oldest
frames to the next older tier (re-pooled), the oldest tier dropping its
oldest: each of tier0.., recent is a ring of frame slots, so only the frames
that change tier move.

Buffer layout (per session, head-major, the attention kernel's layout):
    [prompt | sink | tier (oldest first) ... | recent | chunk]
each segment padded to a multiple of 128 tokens; frames are frame-major then
row-major inside a segment; in the chunk, audio follows video.

A session spec is any object with the attributes of ``workloads.SessionSpec``
(n_heads, head_dim, rope_split, rope_base, grid_h, grid_w, prompt_len,
context_video_tokens, sink_frames, tiers, chunk_video_tokens,
chunk_audio_tokens, latent_fps, audio_rate).
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence

import numpy as np
import torch

from . import capi

TILE = capi.SR_TILE


def _mark(marks, i: int, stream) -> None:
    """Record event i of an optional (before, after) pair on `stream`."""
    if marks is not None:
        marks[i].record(stream if stream is not None else torch.cuda.current_stream())


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def _frame_sizes(total: int, per: int) -> List[int]:
    full, rem = divmod(total, per)
    return [per] * full + ([rem] if rem else [])


class SessionPlan:
    """Per-session structure of the window (host side, no device work)."""

    def __init__(self, spec):
        self.spec = spec
        self.H, self.D = int(spec.n_heads), int(spec.head_dim)
        self.gh, self.gw = int(spec.grid_h), int(spec.grid_w)
        self.frame_tokens = self.gh * self.gw
        ctx = _frame_sizes(int(spec.context_video_tokens), self.frame_tokens)
        n = len(ctx)
        roles = []
        i = 0
        for _ in range(min(int(spec.sink_frames), n)):
            roles.append(("sink", 1, 1))
            i += 1
        for ti, (nf, ph, pw) in enumerate(spec.tiers):
            for _ in range(nf):
                if i >= n:
                    raise ValueError("more tier frames than context frames")
                roles.append((f"tier{ti}", int(ph), int(pw)))
                i += 1
        roles += [("recent", 1, 1)] * (n - i)
        # (segment, t, pool_h, pool_w, source tokens)
        self.context = [(roles[f][0], float(f - n), roles[f][1], roles[f][2], ctx[f]) for f in range(n)]
        self.segments = ["prompt"]
        if any(r == "sink" for r, *_ in self.context):
            self.segments.append("sink")
        self.segments += [f"tier{t}" for t in range(len(spec.tiers))]
        if any(r == "recent" for r, *_ in self.context):
            self.segments.append("recent")
        self.segments.append("chunk")
        self.lengths = {s: 0 for s in self.segments}
        self.lengths["prompt"] = int(spec.prompt_len)
        for role, _, ph, pw, ntok in self.context:
            if role.startswith("tier"):
                if ntok != self.frame_tokens:
                    raise ValueError("pooled frames must be complete")
                self.lengths[role] += self.cells(ph, pw)
            else:
                self.lengths[role] += ntok
        self.chunk_len = int(spec.chunk_video_tokens) + int(spec.chunk_audio_tokens)
        self.lengths["chunk"] = self.chunk_len

    def cells(self, ph: int, pw: int) -> int:
        return _ceil_div(self.gh, ph) * _ceil_div(self.gw, pw)

    def grid_positions(self, t: float, n: int) -> np.ndarray:
        """(t, row, col) of the first n tokens of a full-resolution frame."""
        r, c = np.divmod(np.arange(n), self.gw)
        return np.stack([np.full(n, t), r, c], axis=1).astype(np.float32)

    def chunk_positions(self) -> np.ndarray:
        sp = self.spec
        parts = [self.grid_positions(float(f), n)
                 for f, n in enumerate(_frame_sizes(int(sp.chunk_video_tokens), self.frame_tokens))]
        na = int(sp.chunk_audio_tokens)
        ta = np.arange(na, dtype=np.float64) * (float(sp.latent_fps) / float(sp.audio_rate))
        parts.append(np.stack([ta, np.zeros(na), np.zeros(na)], axis=1).astype(np.float32))
        return np.concatenate(parts).reshape(-1, 3)


class StreamingWindow:
    """Device state of a batch of streaming sessions for one DiT layer.

    All sessions share the segment names and capacities (the largest valid
    length per segment, rounded up to 128); their valid lengths may differ
    (ragged batch).  Buffers are allocated once, zero-filled, and updated in
    place afterwards.
    """

    def __init__(self, specs: Sequence, device="cuda", qk_norm=None):
        """qk_norm: optional (gamma_q, gamma_k, eps) -- per-head RMSNorm gains
        (fp32 [head_dim]) applied to queries and keys before RoPE.  With it
        the window keeps keys before normalisation (pooling then averages the
        projected latents) and every rotation normalises first, fused in one
        kernel."""
        self.plans = [SessionPlan(s) for s in specs]
        p0 = self.plans[0]
        self.B, self.H, self.D = len(self.plans), p0.H, p0.D
        self.split = tuple(int(x) for x in p0.spec.rope_split)
        self.base = float(p0.spec.rope_base)
        for p in self.plans:
            if (p.H, p.D, p.segments, tuple(p.spec.rope_split)) != (self.H, self.D, p0.segments, self.split):
                raise ValueError("sessions of one window must share heads, head_dim, RoPE split and segments")
        self.segments = p0.segments
        self.caps = [max(TILE, _ceil_div(max(p.lengths[s] for p in self.plans), TILE) * TILE)
                     for s in self.segments]
        self.offsets = [int(x) for x in np.cumsum([0] + self.caps[:-1])]
        self.cap_total = int(sum(self.caps))
        self.seg = {s: (int(o), int(c)) for s, o, c in zip(self.segments, self.offsets, self.caps)}
        self.q_cap = max(p.chunk_len for p in self.plans)
        self.device = torch.device(device)
        B, H, D, C = self.B, self.H, self.D, self.cap_total
        kw = dict(device=self.device)
        self.k_raw = torch.zeros(B, H, C, D, dtype=torch.bfloat16, **kw)
        self.k_att = torch.zeros(B, H, C, D, dtype=torch.bfloat16, **kw)
        self.v = torch.zeros(B, H, C, D, dtype=torch.bfloat16, **kw)
        self.pos = torch.zeros(B, C, 3, dtype=torch.float32, **kw)
        self.q_att = torch.zeros(B, H, self.q_cap, D, dtype=torch.bfloat16, **kw)
        self.o = torch.zeros(B, self.q_cap, H, D, dtype=torch.bfloat16, **kw)
        self.lse = torch.zeros(B, H, self.q_cap, dtype=torch.float32, **kw)
        self.status = torch.zeros(1, dtype=torch.int32, **kw)
        # stream clock: t of the current chunk's first latent frame on the
        # time axis every rotation shares (template t + clock)
        self.clock = torch.zeros(1, dtype=torch.float64, **kw)
        ws = capi.sr_chunk_attention_workspace_bytes(B, H, D, self.q_cap) if self.device.type == "cuda" else 0
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, **kw) if ws else None
        lens = np.array([[p.lengths[s] for s in self.segments] for p in self.plans], dtype=np.int32)
        self.lengths = lens
        self.kv_len = torch.from_numpy(lens).to(self.device)
        self.seg_valid = torch.from_numpy(np.ascontiguousarray(lens.T)).to(self.device)   # [n_seg, B]
        self.q_len = torch.tensor([p.chunk_len for p in self.plans], dtype=torch.int32, device=self.device)
        qpos = np.zeros((B, self.q_cap, 3), dtype=np.float32)
        for b, p in enumerate(self.plans):
            qpos[b, :p.chunk_len] = p.chunk_positions()
        self.q_pos = torch.from_numpy(qpos).to(self.device)
        self.scale = 1.0 / math.sqrt(D)
        self.qk_norm = None
        if qk_norm is not None:
            gq, gk, eps = qk_norm
            self.qk_norm = (torch.as_tensor(gq, dtype=torch.float32).to(self.device).contiguous(),
                            torch.as_tensor(gk, dtype=torch.float32).to(self.device).contiguous(), float(eps))

    # ---------------------------------------------------------------- views
    def seg_view(self, buf: torch.Tensor, name: str) -> torch.Tensor:
        """[B, cap, H, D] token-major view of one segment of a head-major buffer."""
        off, cap = self.seg[name]
        return buf[:, :, off:off + cap].permute(0, 2, 1, 3)

    def valid_mask(self, b: int) -> np.ndarray:
        m = np.zeros(self.cap_total, dtype=bool)
        for s, (off, _) in self.seg.items():
            m[off:off + self.plans[b].lengths[s]] = True
        return m

    # ---------------------------------------------------------------- window fill
    def load_window(self, inputs: Sequence, stream=None) -> None:
        """Fill prompt and context segments of every session from its drawn
        inputs (``workloads.SessionInputs``-like: prompt_k/v [Lp, H, D], ctx_k/v
        lists of [tokens, H, D] full-resolution frames, oldest first).  Tier
        frames are pooled on the device by sr_history_compress."""
        dev = self.device
        if hasattr(self, "rings"):   # a reload restarts the window slide
            self.pos = self._pos_loaded
            del self.rings
        self.__dict__.pop("_step_graphs", None)   # captured against the old ring state and position tables
        for b, (plan, inp) in enumerate(zip(self.plans, inputs)):
            kb, vb, pb = self.k_raw[b:b + 1], self.v[b:b + 1], self.pos[b:b + 1]
            lp = plan.lengths["prompt"]
            if lp:
                capi.sr_kv_append(kb, vb, pb, self.seg["prompt"][0], inp.prompt_k.to(dev)[None],
                                  inp.prompt_v.to(dev)[None], torch.zeros(1, lp, 3, device=dev), stream=stream)
            fill = {s: 0 for s in self.segments}
            f = 0
            ctx = plan.context
            while f < len(ctx):
                role, t, ph, pw, ntok = ctx[f]
                if role.startswith("tier"):
                    g = f
                    while g < len(ctx) and ctx[g][0] == role:
                        g += 1
                    nf = g - f
                    cells = plan.cells(ph, pw)
                    src_k = torch.stack([inp.ctx_k[i] for i in range(f, g)]).to(dev)[None]
                    src_v = torch.stack([inp.ctx_v[i] for i in range(f, g)]).to(dev)[None]
                    off = self.seg[role][0] + fill[role]
                    n_out = nf * cells
                    out_k = self.k_raw[b:b + 1, :, off:off + n_out].permute(0, 2, 1, 3).reshape(1, nf, cells, self.H, self.D)
                    out_v = self.v[b:b + 1, :, off:off + n_out].permute(0, 2, 1, 3).reshape(1, nf, cells, self.H, self.D)
                    frame_t = torch.tensor([[ctx[i][1] for i in range(f, g)]], dtype=torch.float32, device=dev)
                    capi.sr_history_compress(src_k, src_v, out_k, out_v, (plan.gh, plan.gw), (ph, pw),
                                             frame_t=frame_t, pos_out=self.pos[b:b + 1, off:off + n_out],
                                             stream=stream)
                    fill[role] += n_out
                    f = g
                else:
                    off = self.seg[role][0] + fill[role]
                    pos = torch.from_numpy(plan.grid_positions(t, ntok)).to(dev)[None]
                    capi.sr_kv_append(kb, vb, pb, off, inp.ctx_k[f].to(dev)[None], inp.ctx_v[f].to(dev)[None],
                                      pos, stream=stream)
                    fill[role] += ntok
                    f += 1
        # chunk positions are the fixed template
        off = self.seg["chunk"][0]
        self.pos[:, off:off + self.q_cap].copy_(self.q_pos)
        # a reload restarts the stream clock; every key of the loaded window is
        # rotated once (padded slots hold zeros and stay zeros)
        self.clock.zero_()
        self._rope(self.k_raw.permute(0, 2, 1, 3), self.k_att.permute(0, 2, 1, 3), self.pos, key=True,
                   stream=stream)

    # ---------------------------------------------------------------- the step
    def append_chunk(self, k: torch.Tensor, v: torch.Tensor, stream=None, rotate: bool = None) -> None:
        """a2 (with a3 of the chunk keys): chunk K and V [B, q_cap, H, D] into
        the chunk segment.  By default the keys are rotated on the way in
        (k_att; the chunk's pre-RoPE keys are never pooled, so k_raw is not
        written); with rotate=False, or with QK normalisation, K goes to
        k_raw unrotated for a later whole-window rotation."""
        if rotate is None:
            rotate = self.qk_norm is None
        off = self.seg["chunk"][0]
        if rotate:
            rot = capi.RopeOut(self.k_att, self.q_pos, self.split, self.base, t_origin=self.clock)
            capi.sr_kv_append(None, self.v, None, off, k, v, None, n_valid=self.q_len, rot=rot, stream=stream)
        else:
            capi.sr_kv_append(self.k_raw, self.v, None, off, k, v, None, n_valid=self.q_len, stream=stream)

    def rotate(self, q: torch.Tensor, stream=None) -> None:
        """a3: RoPE of the chunk queries into q_att, and of the keys whose
        template places float with the chunk: the prefix (prompt, sink), one
        launch over its contiguous slots.  With QK normalisation every window
        key is normalised and rotated again instead (from k_raw)."""
        self._rope(q, self.q_att.permute(0, 2, 1, 3), self.q_pos, key=False, n_valid=self.q_len, stream=stream)
        if self.qk_norm is None:
            self.rotate_prefix(stream)
        else:
            self.rotate_keys(stream)

    def prefix_slots(self) -> int:
        """Slots of the prefix segments (prompt, then sink) at the buffer start."""
        return sum(c for name, c in zip(self.segments, self.caps) if name in ("prompt", "sink"))

    def rotate_prefix(self, stream=None) -> None:
        """RoPE of the prefix slots (prompt, sink) from k_raw into k_att at the
        current clock (one launch)."""
        n = self.prefix_slots()
        self._rope(self.k_raw[:, :, :n].permute(0, 2, 1, 3), self.k_att[:, :, :n].permute(0, 2, 1, 3),
                   self.pos[:, :n], key=True, stream=stream)

    def rotate_keys(self, stream=None) -> None:
        """RoPE of every window slot from k_raw into k_att at the current clock
        (one launch)."""
        self._rope(self.k_raw.permute(0, 2, 1, 3), self.k_att.permute(0, 2, 1, 3), self.pos, key=True,
                   stream=stream)

    def _rope(self, x, y, pos, key: bool, n_valid=None, stream=None) -> None:
        if self.qk_norm is None:
            capi.sr_rope3d_apply(x, y, pos, self.split, self.base, n_valid=n_valid, t_origin=self.clock,
                                 stream=stream)
        else:
            gq, gk, eps = self.qk_norm
            capi.sr_qknorm_rope3d_apply(x, y, gk if key else gq, eps, pos, self.split, self.base, n_valid=n_valid,
                                        t_origin=self.clock, stream=stream)

    def attend(self, stream=None, out: torch.Tensor = None, marks=None) -> torch.Tensor:
        """a4: fused chunk attention -> o [B, q_cap, H, D] (and lse); `out`
        optionally replaces the window's own output buffer; `marks`, a pair
        of CUDA events, is recorded around the launch (for timing)."""
        o = self.o if out is None else out
        _mark(marks, 0, stream)
        capi.sr_chunk_attention_fwd(self.q_att, self.k_att, self.v, o, self.lse, self.caps, self.kv_len,
                                    self.q_len, self.scale, self.status, workspace=self.workspace, stream=stream)
        _mark(marks, 1, stream)
        return o

    def step(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, stream=None,
             out: torch.Tensor = None, marks=None) -> torch.Tensor:
        """One streaming attention step: a2 -> a3 -> a4 (device tensors
        [B, q_cap, H, D], token-major, pre-RoPE)."""
        self.append_chunk(k, v, stream)
        self.rotate(q, stream)
        return self.attend(stream, out=out, marks=marks)

    def step_from_host(self, q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor,
                       o_host: torch.Tensor, staging=None, stream=None) -> torch.Tensor:
        """The streaming step for callers holding host tensors: copy the chunk's
        q, k, v [B, q_cap, H, D] (pinned host memory for asynchronous copies)
        to the device, run the step, copy o back into ``o_host``.  ``staging``
        is an optional (q, k, v) triple of device tensors reused across calls.
        Asynchronous on the current stream; synchronise before reading o_host."""
        if staging is None:
            staging = tuple(torch.empty_like(t, device=self.device) for t in (q_host, k_host, v_host))
        for dst, src in zip(staging, (q_host, k_host, v_host)):
            dst.copy_(src, non_blocking=True)
        o = self.step(*staging, stream=stream)
        o_host.copy_(o, non_blocking=True)
        return o_host

    # ---------------------------------------------------------------- prefix / moving part
    # "StreamRender-H3" (molayo1419.me), streaming context section: the fixed
    # prefix (conditions, reference, sink) is cached once per denoising step
    # and attends only to itself; the moving part (recent history and the
    # current chunk) is recomputed each step and attends to the whole window.
    # A separate cache per denoising step ("bank") is a separate batch entry.
    def prefix_positions(self) -> np.ndarray:
        """[B, prefix_cap, 3] positions of the prefix queries: prompt (0) then sink tokens."""
        lens = [p.lengths["prompt"] + p.lengths.get("sink", 0) for p in self.plans]
        out = np.zeros((self.B, max(lens), 3), dtype=np.float32)
        for b, p in enumerate(self.plans):
            sink = [(t, n) for role, t, _, _, n in p.context if role == "sink"]
            rows = [np.zeros((p.lengths["prompt"], 3), np.float32)] + [p.grid_positions(t, n) for t, n in sink]
            x = np.concatenate(rows)
            out[b, :x.shape[0]] = x
        return out

    def _scratch(self, key: str, n_q: int):
        """Per-shape buffers of the prefix / moving attention, allocated once:
        q_att [B, H, n_q, D], o [B, n_q, H, D], lse, the split workspace."""
        cache = self.__dict__.setdefault("_scratch_bufs", {})
        if (key, n_q) not in cache:
            B, H, D, dev = self.B, self.H, self.D, self.device
            ws_bytes = capi.sr_chunk_attention_workspace_bytes(B, H, D, n_q)
            cache[(key, n_q)] = (torch.zeros(B, H, n_q, D, dtype=torch.bfloat16, device=dev),
                                 torch.zeros(B, n_q, H, D, dtype=torch.bfloat16, device=dev),
                                 torch.zeros(B, H, n_q, dtype=torch.float32, device=dev),
                                 torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev) if ws_bytes else None)
        return cache[(key, n_q)]

    def attend_prefix(self, q_prefix: torch.Tensor, stream=None) -> torch.Tensor:
        """Prefix-self attention: queries of the prefix tokens (prompt, then
        sink), token-major [B, prefix_cap, H, D] before RoPE, over the prefix
        keys only.  Returns o [B, prefix_cap, H, D] (rows past a session's
        prefix length are left alone; the buffer is reused by later calls)."""
        B, n_pre, H, D = q_prefix.shape
        if not hasattr(self, "_prefix_meta"):
            pos = torch.from_numpy(self.prefix_positions()).to(self.device)
            lens = torch.tensor([p.lengths["prompt"] + p.lengths.get("sink", 0) for p in self.plans],
                                dtype=torch.int32, device=self.device)
            kv_len = self.kv_len.clone()
            for si, name in enumerate(self.segments):
                if name not in ("prompt", "sink"):
                    kv_len[:, si] = 0
            self._prefix_meta = (pos, lens, kv_len)
        pos, lens, kv_len = self._prefix_meta
        assert n_pre == pos.shape[1], "q_prefix must cover prompt + sink tokens"
        q_att, o, lse, ws = self._scratch("prefix", n_pre)
        self.rotate_prefix(stream)
        self._rope(q_prefix, q_att.permute(0, 2, 1, 3), pos, key=False, n_valid=lens, stream=stream)
        capi.sr_chunk_attention_fwd(q_att, self.k_att, self.v, o, lse, self.caps, kv_len, lens, self.scale,
                                    self.status, workspace=ws, stream=stream)
        self.prefix_lse = lse
        return o

    def step_moving(self, q_recent: torch.Tensor, k_recent: torch.Tensor, v_recent: torch.Tensor,
                    q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, stream=None, marks=None) -> torch.Tensor:
        """The moving part of one denoising step: the recent frames' recomputed
        K (before RoPE) and V replace the recent segment, the chunk's K and V
        the chunk segment, and the queries of the recent frames followed by
        the chunk attend to the whole window.  Recent tensors [B, n_recent,
        H, D] (every session the same n_recent), chunk tensors as in step().
        Returns o [B, n_recent + q_cap, H, D] (a buffer reused by later calls)."""
        B, n_rec, H, D = q_recent.shape
        off_r, _ = self.seg["recent"]
        if any(p.lengths["recent"] != n_rec for p in self.plans):
            raise ValueError("every session must hold n_recent recent tokens")
        # after window slides the recent frames sit in ring order: write each
        # run of consecutive slots with one append, read positions likewise
        ft = self.plans[0].frame_tokens
        order = self.recent_slot_order()
        runs, j = [], 0
        while j < len(order):
            m = 1
            while j + m < len(order) and order[j + m] == order[j] + m:
                m += 1
            runs.append((order[j], j, m))
            j += m
        for slot, j, m in runs:
            rows = slice(j * ft, min((j + m) * ft, n_rec))
            capi.sr_kv_append(self.k_raw, self.v, None, off_r + slot * ft, k_recent[:, rows], v_recent[:, rows],
                              None, stream=stream)
        self.append_chunk(k, v, stream, rotate=False)
        n_mov = n_rec + self.q_cap
        q_att, o, lse, ws = self._scratch("moving", n_mov)
        # chunk queries straight into their rows of the moving query buffer
        self._rope(q, q_att[:, :, n_rec:].permute(0, 2, 1, 3), self.q_pos, key=False, n_valid=self.q_len,
                   stream=stream)
        self.rotate_keys(stream)
        if len(runs) == 1:
            pos_r = self.pos[:, off_r:off_r + n_rec]
        else:   # a wrapped ring holds whole frames only
            pos_r = torch.cat([self.pos[:, off_r + slot * ft:off_r + (slot + m) * ft] for slot, _, m in runs], dim=1)
        self._rope(q_recent, q_att[:, :, :n_rec].permute(0, 2, 1, 3), pos_r, key=False, stream=stream)
        if not hasattr(self, "_moving_q_len") or self._moving_q_len[0] != n_rec:
            self._moving_q_len = (n_rec, self.q_len + n_rec)
        _mark(marks, 0, stream)
        capi.sr_chunk_attention_fwd(q_att, self.k_att, self.v, o, lse, self.caps, self.kv_len,
                                    self._moving_q_len[1], self.scale, self.status, workspace=ws, stream=stream)
        _mark(marks, 1, stream)
        self.moving_lse = lse
        return o

    def check_status(self) -> None:
        """Raise if a bounded wait inside the attention kernel gave up
        (synchronises with the device)."""
        s = int(self.status.item())
        if s != 0:
            self.status.zero_()
            raise capi.SrError("sr_chunk_attention_fwd", s, "a pipeline wait timed out on the device")

    def tier_boundaries(self):
        """(source segment, destination tier, source grid, pool) for every tier
        boundary, destination-oldest first: each tier is fed by the next
        newer tier, the newest tier by the recent frames."""
        plan = self.plans[0]
        tiers = [f"tier{i}" for i in range(len(plan.spec.tiers))]
        if not tiers or "recent" not in self.segments:
            return []
        grid = {"recent": (plan.gh, plan.gw)}
        for i, (_, ph, pw) in enumerate(plan.spec.tiers):
            grid[tiers[i]] = (_ceil_div(plan.gh, ph), _ceil_div(plan.gw, pw))
        out = []
        for i, dst in enumerate(tiers):
            src = tiers[i + 1] if i + 1 < len(tiers) else "recent"
            (gh, gw), (dh, dw) = grid[src], grid[dst]
            out.append((src, dst, (gh, gw), (_ceil_div(gh, dh), _ceil_div(gw, dw))))
        return out

    # ---------------------------------------------------------------- window slide
    # After a chunk is finished its clean frames become the newest context;
    # every tier hands its oldest frames to the next older tier, pooled once
    # more, and the oldest tier drops its oldest frames.  The sink stays.
    # Each of tier0.., recent is a ring of frame slots with a pointer to its
    # oldest frame, so nothing is moved but the frames that change tier; the
    # window template (t of a frame = its rank in the window) is rewritten by
    # switching to a precomputed position table of the new ring state.
    MAX_PHASES = 64

    def _ring_setup(self, n: int) -> None:
        """Host side of the rings for slides of n frames: per ring its slot
        count, tokens per frame, template t of its oldest frame; the pointer
        state starts at 0 (load_window fills slots in chronological order)."""
        plan = self.plans[0]
        if any(p.context != plan.context for p in self.plans):
            raise ValueError("the window slide needs sessions with the same context structure")
        rings = {}
        for role, t, ph, pw, ntok in plan.context:
            if role == "sink":
                continue
            if ntok != plan.frame_tokens:
                raise ValueError("the window slide needs whole history frames")
            tok = plan.cells(ph, pw) if role.startswith("tier") else plan.frame_tokens
            r = rings.setdefault(role, {"frames": 0, "tok": tok, "t0": t})
            r["frames"] += 1
        if "recent" not in rings or any(n > r["frames"] for r in rings.values()):
            raise ValueError(f"a slide of {n} frames must fit in every history ring "
                             f"({ {k: r['frames'] for k, r in rings.items()} })")
        self.rings, self.slide_frames = rings, n
        self.ring_ptr = {k: 0 for k in rings}
        # each pointer moves n slots per slide: F / gcd(F, n) states per ring
        self.period = math.lcm(*[r["frames"] // math.gcd(r["frames"], n) for r in rings.values()])

    def ring_positions(self, ptr) -> np.ndarray:
        """[cap_total, 3] template positions of the history ring slots for
        pointer state ``ptr`` (other rows zero): t from the frame's rank in its
        ring, (h, w) its grid cell or its cell's member mean."""
        plan = self.plans[0]
        pos = np.zeros((self.cap_total, 3), dtype=np.float32)
        for role, r in self.rings.items():
            off = self.seg[role][0]
            if role.startswith("tier"):
                _, ph, pw = plan.spec.tiers[int(role[4:])]
                cells = []
                for ci in range(_ceil_div(plan.gh, ph)):
                    for cj in range(_ceil_div(plan.gw, pw)):
                        r0, r1 = ci * ph, min((ci + 1) * ph, plan.gh)
                        c0, c1 = cj * pw, min((cj + 1) * pw, plan.gw)
                        cells.append((0.5 * (r0 + r1 - 1), 0.5 * (c0 + c1 - 1)))
                hw = np.asarray(cells, dtype=np.float32)
            else:
                hw = plan.grid_positions(0.0, plan.frame_tokens)[:, 1:]
            for slot in range(r["frames"]):
                rank = (slot - ptr[role]) % r["frames"]
                rows = slice(off + slot * r["tok"], off + (slot + 1) * r["tok"])
                pos[rows, 0] = r["t0"] + rank
                pos[rows, 1:] = hw
        return pos

    def slide_ops(self, ptr):
        """Kernel calls of one slide from pointer state ``ptr`` (host only):
        ("pool", src, src_frame, dst, dst_frame, m, grid, pool) and
        ("append", recent_frame, clean_frame, m), in launch order, and the
        next pointer state.  Boundaries run oldest tier first, so a ring's
        oldest frames are read before the next boundary overwrites them."""
        n = self.slide_frames
        ops, nxt = [], dict(ptr)
        for src, dst, grid, pool in self.tier_boundaries():
            rs, rd = self.rings[src], self.rings[dst]
            done = 0
            while done < n:   # split where either ring wraps around
                fs = (ptr[src] + done) % rs["frames"]
                fd = (ptr[dst] + done) % rd["frames"]
                m = min(n - done, rs["frames"] - fs, rd["frames"] - fd)
                ops.append(("pool", src, fs, dst, fd, m, grid, pool))
                done += m
            nxt[dst] = (ptr[dst] + n) % rd["frames"]
        rr = self.rings["recent"]
        done = 0
        while done < n:
            fr = (ptr["recent"] + done) % rr["frames"]
            m = min(n - done, rr["frames"] - fr)
            ops.append(("append", fr, done, m))
            done += m
        nxt["recent"] = (ptr["recent"] + n) % rr["frames"]
        return ops, nxt

    def _ring_frames(self, buf, role: str, first: int, n: int) -> torch.Tensor:
        """[B, n, tok, H, D] view of n consecutive frame slots of a ring."""
        r = self.rings[role]
        off = self.seg[role][0] + first * r["tok"]
        return buf[:, :, off:off + n * r["tok"]].permute(0, 2, 1, 3).reshape(self.B, n, r["tok"], self.H, self.D)

    def _phase_tables(self) -> None:
        """Device position tables of every pointer state the slides cycle
        through (the sink, prompt and chunk rows copied from the loaded window)."""
        if self.period > self.MAX_PHASES:
            raise ValueError(f"ring period {self.period} > {self.MAX_PHASES} position tables")
        ctx = [self.seg[r] for r in self.rings]
        lo, hi = min(o for o, _ in ctx), max(o + c for o, c in ctx)
        self._pos_loaded = self.pos
        self._phases, ptr = {}, dict(self.ring_ptr)
        for _ in range(self.period):
            tab = self._pos_loaded.clone()
            tab[:, lo:hi] = torch.from_numpy(self.ring_positions(ptr)[lo:hi]).to(self.device)
            self._phases[tuple(ptr.values())] = tab
            ptr = self.slide_ops(ptr)[1]

    def advance(self, k_clean: torch.Tensor, v_clean: torch.Tensor, stream=None) -> None:
        """Slide the window by the finished chunk (a1 in streaming use).

        k_clean, v_clean: the chunk's clean video frames, token-major
        [B, n * frame_tokens, H, D], K before RoPE (every session the same n,
        at most every ring's frame count).  Launches one
        sr_history_compress per tier boundary (two where a ring wraps) and
        one sr_kv_append (two on a wrap); positions switch to the new state's
        table (no copy); the next rotate() re-positions the keys."""
        plan = self.plans[0]
        n = k_clean.shape[1] // plan.frame_tokens
        if n < 1 or n * plan.frame_tokens != k_clean.shape[1] or v_clean.shape != k_clean.shape:
            raise ValueError("clean K/V must hold whole frames")
        if not hasattr(self, "rings"):
            self._ring_setup(n)
            self._phase_tables()
        elif n != self.slide_frames:
            raise ValueError(f"every slide must move {self.slide_frames} frames")
        ops, nxt = self.slide_ops(self.ring_ptr)
        self.ring_ptr = nxt
        self.pos = self._phases[tuple(nxt.values())]   # the new state's template: the entering keys' places
        capi.sr_stream_clock_advance(self.clock, float(n), stream=stream)
        self._launch_slide(ops, k_clean, v_clean, stream)

    def _launch_slide(self, ops, k_clean, v_clean, stream=None) -> None:
        """The kernel calls of one slide plan (no host state changes).  The
        keys entering a ring slot are rotated on the way in at the template
        of self.pos (the new ring state) plus the clock, except with QK
        normalisation, whose every step re-rotates the whole window."""
        ft = self.plans[0].frame_tokens
        rotate = self.qk_norm is None
        for op in ops:
            if op[0] == "pool":
                _, src, fs, dst, fd, m, grid, pool = op
                rot = None
                if rotate:
                    r = self.rings[dst]
                    off = self.seg[dst][0] + fd * r["tok"]
                    rot = capi.RopeOut(self._ring_frames(self.k_att, dst, fd, m), self.pos[:, off:off + m * r["tok"]],
                                       self.split, self.base, t_origin=self.clock)
                capi.sr_history_compress(self._ring_frames(self.k_raw, src, fs, m),
                                         self._ring_frames(self.v, src, fs, m),
                                         self._ring_frames(self.k_raw, dst, fd, m),
                                         self._ring_frames(self.v, dst, fd, m), grid, pool, rot=rot, stream=stream)
            else:
                _, fr, fc, m = op
                off = self.seg["recent"][0] + fr * ft
                rot = capi.RopeOut(self.k_att, self.pos[:, off:off + m * ft], self.split, self.base,
                                   t_origin=self.clock) if rotate else None
                capi.sr_kv_append(self.k_raw, self.v, None, off, k_clean[:, fc * ft:(fc + m) * ft],
                                  v_clean[:, fc * ft:(fc + m) * ft], None, rot=rot, stream=stream)

    def step_ops(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, k_clean: torch.Tensor = None,
                 v_clean: torch.Tensor = None, ptr=None):
        """The library calls of one streaming step before the attention, in
        launch order: (name, algorithmic bytes, branch, launch) with launch()
        issuing the call on the current stream.  With k_clean / v_clean the
        stream clock advance and the window slide from ring state ``ptr`` come
        first (its pooling and append calls); then the chunk append, the RoPE
        of the chunk queries and the RoPE of the prefix (or, with QK
        normalisation, of the whole window).  Algorithmic bytes count each
        valid token's data read or written once (positions included where a
        call reads them), the measure of the HBM roofline of each call.
        Branch 0 runs first; the calls of branches 1, 2, ... depend only on
        branch 0 and on earlier calls of their own branch, so the branches may
        run concurrently (a last branch 4, the whole-window RoPE, waits for
        all the others)."""
        H, D, B = self.H, self.D, self.B
        row = H * D * 2                                   # bytes of one token's K (or V) row
        fused = self.qk_norm is None                      # keys rotated on entry (else re-rotated every step)
        out_rows = 3 if fused else 2                      # K before RoPE, K rotated, V
        ops = []
        if k_clean is not None:
            ft = self.plans[0].frame_tokens
            n = self.slide_frames
            ops.append(("stream clock", None, 0, lambda: capi.sr_stream_clock_advance(self.clock, float(n))))
            for op in self.slide_ops(ptr)[0]:
                if op[0] == "pool":
                    _, src, _, dst, _, m, _, _ = op
                    t_src, t_dst = m * self.rings[src]["tok"], m * self.rings[dst]["tok"]
                    nb = B * (2 * t_src * row + out_rows * t_dst * row + (12 * t_dst if fused else 0))
                    ops.append((f"pool {src}->{dst}", nb, 1,
                                lambda op=op: self._launch_slide([op], k_clean, v_clean)))
                else:
                    t = op[3] * ft
                    nb = B * (2 * t * row + out_rows * t * row + (12 * t if fused else 0))
                    ops.append(("append clean frames", nb, 1,
                                lambda op=op: self._launch_slide([op], k_clean, v_clean)))
        n_q = int(sum(p.chunk_len for p in self.plans))
        ops.append(("append chunk" + (" + RoPE" if fused else ""), 2 * 2 * n_q * row + (12 * n_q if fused else 0),
                    2, lambda: self.append_chunk(k, v)))
        ops.append(("rope chunk queries", n_q * (2 * row + 12), 3,
                    lambda: self._rope(q, self.q_att.permute(0, 2, 1, 3), self.q_pos, key=False, n_valid=self.q_len)))
        if fused:
            n_pre = int(sum(p.lengths["prompt"] + p.lengths.get("sink", 0) for p in self.plans))
            ops.append(("rope prefix keys", n_pre * (2 * row + 12), 3, lambda: self.rotate_prefix()))
        else:   # every key is re-rotated from k_raw: after the slide and the chunk append
            n_keys = int(self.lengths.sum())
            ops.append(("rope window keys", n_keys * (2 * row + 12), 4, lambda: self.rotate_keys()))
        return ops

    def _launch_branches(self, ops) -> None:
        """Issue step_ops entries: branch 0 on the current stream, every other
        branch on a side stream forked from it (joined back at the end);
        branch 4 (the whole-window RoPE) also waits for every other branch.
        Captured into a CUDA graph, the branches become parallel paths the
        device may run at the same time."""
        cur = torch.cuda.current_stream()
        for _, _, br, launch in ops:
            if br == 0:
                launch()
        side = self.__dict__.setdefault("_side_streams", {})
        ends = []
        for b in sorted({br for _, _, br, _ in ops if br > 0}):
            st = side.setdefault(b, torch.cuda.Stream(device=self.device))
            st.wait_stream(cur)
            if b == 4:
                for e in ends:
                    st.wait_stream(e)
            with torch.cuda.stream(st):
                for _, _, br, launch in ops:
                    if br == b:
                        launch()
            ends.append(st)
        for st in ends:
            cur.wait_stream(st)

    def graph_step(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, k_clean: torch.Tensor = None,
                   v_clean: torch.Tensor = None, marks=None, op_marks=None) -> torch.Tensor:
        """advance(k_clean, v_clean) (when given) and step(q, k, v), replayed
        from CUDA graphs: no per-launch host work, and the launches follow
        each other without gaps.

        The tensors must be the same (addresses) on every call.  Each ring
        state is captured the first time it occurs, after that call has run
        eagerly; later calls replay two graphs on the current stream (the
        slide, append and RoPE; the attention), with `marks` recorded around
        the second.  In the first graph the independent calls (see step_ops)
        are parallel branches.  ``op_marks`` (a list the call fills) instead
        replays every call of the step from a graph of its own, one after the
        other, with a CUDA event recorded before each and after the attention:
        it receives (name, algorithmic bytes, start event, end event) per call
        and ("attention", None, start, end) last -- the per-call timing of the
        step.  Returns the window's output buffer."""
        slide = k_clean is not None
        key = tuple(self.ring_ptr.values()) if slide and hasattr(self, "rings") else None
        graphs = self.__dict__.setdefault("_step_graphs", {})
        if key not in graphs:
            if slide:
                self.advance(k_clean, v_clean)
            self.step(q, k, v, marks=marks)
            torch.cuda.synchronize()
            if slide and key is None:    # the rings were set up by this first slide: capture from the next one
                return self.o
            ops = self.step_ops(q, k, v, k_clean, v_clean, dict(zip(self.rings, key)) if slide else None)
            g_prep, g_attn = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_prep):   # self.pos already holds the next state's table
                self._launch_branches(ops)
            with torch.cuda.graph(g_attn):
                self.attend()
            per_op = []
            for name, nbytes, _, launch in ops:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    launch()
                per_op.append((name, nbytes, g))
            graphs[key] = (g_prep, g_attn, per_op)
            return self.o
        g_prep, g_attn, per_op = graphs[key]
        if slide:
            nxt = self.slide_ops(self.ring_ptr)[1]
            self.ring_ptr = nxt
            self.pos = self._phases[tuple(nxt.values())]
        if op_marks is None:
            g_prep.replay()
            _mark(marks, 0, None)
            g_attn.replay()
            _mark(marks, 1, None)
            return self.o
        stream = torch.cuda.current_stream()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(per_op) + 2)]
        for i, (_, _, g) in enumerate(per_op):
            evs[i].record(stream)
            g.replay()
        evs[-2].record(stream)
        g_attn.replay()
        evs[-1].record(stream)
        op_marks.extend((name, nbytes, evs[i], evs[i + 1]) for i, (name, nbytes, _) in enumerate(per_op))
        op_marks.append(("attention", None, evs[-2], evs[-1]))
        return self.o

    def recent_slot_order(self) -> List[int]:
        """Recent frames in chronological order -> their ring slots."""
        if not hasattr(self, "rings"):
            return list(range(_ceil_div(self.plans[0].lengths.get("recent", 0), self.plans[0].frame_tokens)))
        r = self.rings["recent"]
        return [(self.ring_ptr["recent"] + j) % r["frames"] for j in range(r["frames"])]

    # ---------------------------------------------------------------- checkpoint / resume
    # "StreamRender-H3" (molayo1419.me), inference acceleration section: the
    # per-layer KV buffers are persistent and updated in place, so a session's
    # whole state is those buffers plus the host-side ring pointers and the
    # position table they select.
    def export_state(self) -> dict:
        """Snapshot of the session state on the host (synchronises with the
        device): the window buffers (keys before and after RoPE, values), the
        stream clock, the position table in use and, once the window has slid,
        the ring pointers,
        the frames per slide and the position table of the loaded window that
        every ring state's table is built from.  ``import_state`` on a window
        made from the same specs continues the stream bit for bit."""
        torch.cuda.synchronize(self.device)
        st = {"shape": (self.B, self.H, self.cap_total, self.D), "segments": list(self.segments),
              "caps": list(self.caps), "lengths": self.lengths.copy(),
              "k_raw": self.k_raw.cpu(), "k_att": self.k_att.cpu(), "v": self.v.cpu(), "pos": self.pos.cpu(),
              "clock": self.clock.cpu()}
        if hasattr(self, "rings"):
            st.update(ring_ptr=dict(self.ring_ptr), slide_frames=int(self.slide_frames),
                      pos_loaded=self._pos_loaded.cpu())
        return st

    def import_state(self, st: dict) -> None:
        """Restore a snapshot taken by ``export_state`` (same specs: shapes,
        segments and valid lengths must agree).  Captured step graphs are
        dropped; the next slide continues from the saved ring pointers."""
        if tuple(st["shape"]) != (self.B, self.H, self.cap_total, self.D) or list(st["segments"]) != \
                list(self.segments) or list(st["caps"]) != list(self.caps) or \
                not np.array_equal(np.asarray(st["lengths"]), self.lengths):
            raise ValueError("the snapshot was taken on a window of another shape or layout")
        self.__dict__.pop("_step_graphs", None)
        for name in ("k_raw", "k_att", "v", "clock"):
            getattr(self, name).copy_(st[name])
        if "ring_ptr" in st:
            self.pos = st["pos_loaded"].to(self.device)
            self._ring_setup(int(st["slide_frames"]))
            self._phase_tables()
            if set(st["ring_ptr"]) != set(self.rings):
                raise ValueError("the snapshot's rings do not match this window")
            self.ring_ptr = {k: int(st["ring_ptr"][k]) for k in self.rings}
            self.pos = self._phases[tuple(self.ring_ptr.values())]
        else:
            if hasattr(self, "rings"):
                del self.rings
            self.pos = torch.zeros_like(self.pos)
            self.pos.copy_(st["pos"])
        torch.cuda.synchronize(self.device)


class HostStepPipeline:
    """Runs consecutive streaming steps for a caller that holds its tensors in
    pinned host memory, overlapping the transfers with the compute: step i+1's
    uploads and step i's download run on a copy stream while step i computes
    on the compute stream.  Two staging sets (q, k, v, o) alternate between
    steps; every step still moves its own inputs and its output.

        pipe = HostStepPipeline(window)
        for q_h, k_h, v_h, o_h in steps:          # pinned host tensors
            pipe.step(q_h, k_h, v_h, o_h)           # asynchronous
        pipe.synchronize()                          # every o_h is now valid

    With ``slide=True`` every step after the first first slides the window
    by the previous step's chunk: the video rows of its K and V (already on
    the device in the previous staging set) become the newest history.
    """

    def __init__(self, window: StreamingWindow, depth: int = 2):
        self.win = window
        dev = window.device
        shape = (window.B, window.q_cap, window.H, window.D)
        self.compute = torch.cuda.current_stream(dev)
        self.copy = torch.cuda.Stream(device=dev)       # uploads
        self.copy_back = torch.cuda.Stream(device=dev)  # downloads (the link is full duplex)
        self.sets = [tuple(torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in range(4))
                     for _ in range(depth)]
        self.free = [torch.cuda.Event() for _ in range(depth)]   # staging set reusable (its download done)
        self.read = [torch.cuda.Event() for _ in range(depth)]   # ... and the slide after it has read its K, V
        self.i = 0

    def step(self, q_h: torch.Tensor, k_h: torch.Tensor, v_h: torch.Tensor, o_h: torch.Tensor,
             slide: bool = False) -> None:
        s = self.i % len(self.sets)
        q, k, v, o = self.sets[s]
        uploaded, computed = torch.cuda.Event(), torch.cuda.Event()
        with torch.cuda.stream(self.copy):
            self.copy.wait_event(self.free[s])
            self.copy.wait_event(self.read[s])
            q.copy_(q_h, non_blocking=True)
            k.copy_(k_h, non_blocking=True)
            v.copy_(v_h, non_blocking=True)
            uploaded.record(self.copy)
        self.compute.wait_event(uploaded)
        if slide and self.i > 0:
            p = (self.i - 1) % len(self.sets)
            _, kp, vp, _ = self.sets[p]
            n = int(self.win.plans[0].spec.chunk_video_tokens)
            self.win.advance(kp[:, :n], vp[:, :n], stream=self.compute)
            self.read[p].record(self.compute)
        self.win.step(q, k, v, stream=self.compute, out=o)
        computed.record(self.compute)
        with torch.cuda.stream(self.copy_back):
            self.copy_back.wait_event(computed)
            o_h.copy_(o, non_blocking=True)
            self.free[s].record(self.copy_back)
        self.i += 1

    def synchronize(self) -> None:
        self.copy.synchronize()
        self.copy_back.synchronize()
        self.compute.synchronize()
