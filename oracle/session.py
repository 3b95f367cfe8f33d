"""Whole-step oracle: window KV assembly, pooling, RoPE and attention in fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The step follows the pages' order: the history tiers are pooled from the
full-resolution frames (pre-RoPE K and V, pooled per head), every token of the
window is placed at its window-relative position, Q and K are rotated, and
each chunk query attends over all valid prompt, context and chunk keys with
scale 1/sqrt(D).  Readings are listed in ``oracle/layout.py`` and below.

Reading on what is pooled: the to_k / to_v projections are linear ("MiniMax-H3
deep dive", tensor-name paragraph), so averaging latent tokens before the
projection equals averaging K and V after it; the oracle averages K and V.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import numpy as np

from . import attention, layout, pool, rms_norm, rope3d, _f64


def pooled_tier(spec, frames_k, frames_v, ph: int, pw: int):
    """Pool full-resolution frames [F x (Gh*Gw, H, D)] -> (K, V) [F*cells, H, D]
    and positions of the cells relative to each frame ((mean row, mean col))."""
    H, D = spec.n_heads, spec.head_dim
    F = len(frames_k)
    xk = np.stack([_f64(f) for f in frames_k]).reshape(F, spec.grid_h, spec.grid_w, H, D)
    xv = np.stack([_f64(f) for f in frames_v]).reshape(F, spec.grid_h, spec.grid_w, H, D)
    pk = pool(xk, ph, pw)
    pv = pool(xv, ph, pw)
    cells = pk.shape[1] * pk.shape[2]
    return pk.reshape(F * cells, H, D), pv.reshape(F * cells, H, D)


def session_kv(spec, inp, heads: Optional[Sequence[int]] = None) -> List[Dict]:
    """Segments in buffer order: dicts with name, k (pre-RoPE), v [n, H', D]
    fp64 and pos [n, 3] fp64, for the selected heads (default all; heads are
    independent, so a subset only skips work)."""
    if heads is not None:
        sel = list(heads)
        inp = type(inp)(inp.prompt_k[:, sel], inp.prompt_v[:, sel], [t[:, sel] for t in inp.ctx_k],
                        [t[:, sel] for t in inp.ctx_v], inp.q[:, sel], inp.k[:, sel], inp.v[:, sel])
        spec = type(spec)(**{**spec.__dict__, "n_heads": len(sel)})
    H, D = spec.n_heads, spec.head_dim
    segs = {name: {"name": name, "k": [], "v": [], "pos": []} for name in layout.segment_names(spec)}
    segs["prompt"]["k"].append(_f64(inp.prompt_k))
    segs["prompt"]["v"].append(_f64(inp.prompt_v))
    segs["prompt"]["pos"] += [(0.0, 0.0, 0.0)] * spec.prompt_len
    for f, (t, role, ph, pw, n) in enumerate(layout.context_plan(spec)):
        s = segs[role]
        if role.startswith("tier"):
            k, v = pooled_tier(spec, [inp.ctx_k[f]], [inp.ctx_v[f]], ph, pw)
            s["k"].append(k)
            s["v"].append(v)
            s["pos"] += [(t, mr, mc) for (_, _, _, _, mr, mc) in
                         layout.pooled_cells(spec.grid_h, spec.grid_w, ph, pw)]
        else:
            s["k"].append(_f64(inp.ctx_k[f]))
            s["v"].append(_f64(inp.ctx_v[f]))
            for i in range(n):
                r, c = layout.frame_token_rc(i, spec.grid_w)
                s["pos"].append((t, float(r), float(c)))
    segs["chunk"]["k"].append(_f64(inp.k))
    segs["chunk"]["v"].append(_f64(inp.v))
    segs["chunk"]["pos"] += layout.chunk_positions(spec)
    out = []
    for name in layout.segment_names(spec):
        s = segs[name]
        k = np.concatenate(s["k"]) if s["k"] else np.zeros((0, H, D))
        v = np.concatenate(s["v"]) if s["v"] else np.zeros((0, H, D))
        pos = np.asarray(s["pos"], dtype=np.float64).reshape(-1, 3)
        assert k.shape[0] == v.shape[0] == pos.shape[0]
        out.append({"name": name, "k": k, "v": v, "pos": pos})
    return out


def session_reference(spec, inp, heads: Optional[Sequence[int]] = None,
                      rows: Optional[Sequence[int]] = None, qk_norm=None):
    """O [n_rows, n_heads_sel, D] and LSE [n_rows, n_heads_sel] in fp64 for the
    chunk queries ``rows`` (default all) and ``heads`` (default all).

    qk_norm: optional (gamma_q, gamma_k, eps).  Reading of the norm_q /
    norm_k tensors ("MiniMax-H3 deep dive", tensor-name paragraph): every
    query and key vector (pooled keys after pooling) is RMS-normalised with
    its gain before RoPE."""
    H, D = spec.n_heads, spec.head_dim
    heads = list(range(H)) if heads is None else list(heads)
    segs = session_kv(spec, inp, heads)
    k_all = np.concatenate([s["k"] for s in segs])
    v_all = np.concatenate([s["v"] for s in segs])
    p_all = np.concatenate([s["pos"] for s in segs])
    if qk_norm is not None:
        k_all = rms_norm(k_all, qk_norm[1], qk_norm[2])
    k_rot = rope3d(k_all, p_all, spec.rope_split, spec.rope_base)
    q = _f64(inp.q)[:, heads]
    if qk_norm is not None:
        q = rms_norm(q, qk_norm[0], qk_norm[2])
    q_pos = np.asarray(layout.chunk_positions(spec), dtype=np.float64)
    if rows is not None:
        rows = list(rows)
        q = q[rows]
        q_pos = q_pos[rows]
    q_rot = rope3d(q, q_pos, spec.rope_split, spec.rope_base)
    scale = 1.0 / np.sqrt(D)
    n = q_rot.shape[0]
    o = np.empty((n, len(heads), D))
    lse = np.empty((n, len(heads)))
    for hi in range(len(heads)):
        o[:, hi], lse[:, hi] = attention(np.ascontiguousarray(q_rot[:, hi]),
                                         np.ascontiguousarray(k_rot[:, hi]),
                                         np.ascontiguousarray(v_all[:, hi]), scale)
    return o, lse


def prefix_reference(spec, inp, mov, heads: Optional[Sequence[int]] = None, rows: Optional[Sequence[int]] = None):
    """Attention of the fixed prefix's own queries (prompt then sink tokens)
    over the prefix keys only.

    Source: "StreamRender-H3" (molayo1419.me), streaming context section: the
    prefix cache (text and image conditions, reference image, sink) is
    computed once per denoising step; the fixed prefix attends only to
    itself, the moving part to the whole window.  Reading: prefix = prompt +
    sink segments; prompt queries unrotated like their keys, sink queries at
    the sink frame's positions."""
    H, D = spec.n_heads, spec.head_dim
    heads = list(range(H)) if heads is None else list(heads)
    segs = {s["name"]: s for s in session_kv(spec, inp, heads)}
    names = [n for n in ("prompt", "sink") if n in segs]
    k = np.concatenate([segs[n]["k"] for n in names])
    v = np.concatenate([segs[n]["v"] for n in names])
    pos = np.concatenate([segs[n]["pos"] for n in names])
    k_rot = rope3d(k, pos, spec.rope_split, spec.rope_base)
    q = _f64(mov.prefix_q)[:, heads]
    q_pos = pos
    if rows is not None:
        q, q_pos = q[list(rows)], q_pos[list(rows)]
    q_rot = rope3d(q, q_pos, spec.rope_split, spec.rope_base)
    scale = 1.0 / np.sqrt(D)
    o = np.empty((q_rot.shape[0], len(heads), D))
    lse = np.empty((q_rot.shape[0], len(heads)))
    for hi in range(len(heads)):
        o[:, hi], lse[:, hi] = attention(np.ascontiguousarray(q_rot[:, hi]), np.ascontiguousarray(k_rot[:, hi]),
                                         np.ascontiguousarray(v[:, hi]), scale)
    return o, lse


def moving_reference(spec, inp, mov, heads: Optional[Sequence[int]] = None, rows: Optional[Sequence[int]] = None):
    """Attention of the moving part's queries (recent frames, then the chunk)
    over the whole window, where the recent frames' keys and values are the
    recomputed ones (only the recent history and the current chunk are
    recomputed at inference; same source as prefix_reference)."""
    H, D = spec.n_heads, spec.head_dim
    heads = list(range(H)) if heads is None else list(heads)
    segs = session_kv(spec, inp, heads)
    for sg in segs:
        if sg["name"] == "recent":
            assert sg["k"].shape[0] == mov.recent_k.shape[0]
            sg["k"] = _f64(mov.recent_k)[:, heads]
            sg["v"] = _f64(mov.recent_v)[:, heads]
            recent_pos = sg["pos"]
    k = np.concatenate([sg["k"] for sg in segs])
    v = np.concatenate([sg["v"] for sg in segs])
    pos = np.concatenate([sg["pos"] for sg in segs])
    k_rot = rope3d(k, pos, spec.rope_split, spec.rope_base)
    q = np.concatenate([_f64(mov.recent_q)[:, heads], _f64(inp.q)[:, heads]])
    q_pos = np.concatenate([recent_pos, np.asarray(layout.chunk_positions(spec), dtype=np.float64)])
    if rows is not None:
        q, q_pos = q[list(rows)], q_pos[list(rows)]
    q_rot = rope3d(q, q_pos, spec.rope_split, spec.rope_base)
    scale = 1.0 / np.sqrt(D)
    o = np.empty((q_rot.shape[0], len(heads), D))
    lse = np.empty((q_rot.shape[0], len(heads)))
    for hi in range(len(heads)):
        o[:, hi], lse[:, hi] = attention(np.ascontiguousarray(q_rot[:, hi]), np.ascontiguousarray(k_rot[:, hi]),
                                         np.ascontiguousarray(v[:, hi]), scale)
    return o, lse


def slide_window(spec, inp, clean_k, clean_v, q, k, v):
    """The session one chunk later: the finished chunk's clean video frames
    (token-major [n * Gh*Gw, H, D]) join the history as its newest frames,
    the n oldest frames after the sink leave it, and the next chunk's q, k, v
    replace the chunk.  Every tier is then pooled afresh from full resolution
    by ``session_kv`` (the definition of the window at that time).

    Reading: "StreamRender-H3" (molayo1419.me), streaming context section --
    the context is the sink plus the most recent outputs, so a finished chunk
    pushes the oldest non-sink frames out; "AlayaRenderer-Flash"
    (aitrends.kr), technical details -- frames age from the recent tier into
    the pooled tiers, oldest tier coarsest."""
    ft = spec.grid_h * spec.grid_w
    n = clean_k.shape[0] // ft
    assert n * ft == clean_k.shape[0] and clean_v.shape == clean_k.shape
    sink = spec.sink_frames
    hist_k = list(inp.ctx_k[sink:]) + [clean_k[i * ft:(i + 1) * ft] for i in range(n)]
    hist_v = list(inp.ctx_v[sink:]) + [clean_v[i * ft:(i + 1) * ft] for i in range(n)]
    keep = len(inp.ctx_k) - sink
    return type(inp)(inp.prompt_k, inp.prompt_v, list(inp.ctx_k[:sink]) + hist_k[-keep:],
                     list(inp.ctx_v[:sink]) + hist_v[-keep:], q, k, v)
