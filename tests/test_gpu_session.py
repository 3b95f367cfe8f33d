"""Whole-step parity on the five workload configs (needs a B200).

The CUDA path runs exactly as the bench runs it (``StreamingWindow``: window
fill with device pooling, then a2 append -> a3 RoPE -> a4 attention); the
oracle recomputes the same step in fp64 from the same seeded inputs.  Full
sizes are checked on sampled (row, head) outputs that include every tile
boundary and the ragged tail; the tiny config is checked in full."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import layout as olayout
import workloads
from streaming_video_audio_b200.window import StreamingWindow
from tests.helpers import ATTN_MAX_ABS, ATTN_MEAN_ABS, LSE_ABS, attn_errors, sample_rows, ulp_diff_bf16

pytestmark = pytest.mark.gpu

# (heads checked per session, random rows per session) for each config
SAMPLING = {1: (None, None), 2: ([0, 17, 39], 96), 3: ([0, 21, 39], 96), 4: ([0, 39], 48), 5: (1, 16)}


def lse_bound(spec, inp, h, rows):
    """End-to-end LSE error bound per row: the rotated q and k are rounded to
    bf16 (relative 2^-9 per component) before the attention, so every score
    moves by at most scale * 2^-8 * |q_i| * max_j |k_j| (rotation preserves
    norms; pooled keys are no longer than the longest member), and the LSE,
    a soft maximum of the scores, by no more; plus the kernel's own 1e-3."""
    q = inp.q[rows, h].double()
    kmax = max(t[:, h].double().norm(dim=-1).max().item()
               for t in [inp.prompt_k, inp.k] + list(inp.ctx_k) if t.shape[0])
    return (2.0 ** -8) * q.norm(dim=-1).numpy() * kmax / math.sqrt(spec.head_dim) + LSE_ABS


def _chunk_tensors(win, inputs):
    B, qc, H, D = win.B, win.q_cap, win.H, win.D
    out = []
    for name in ("q", "k", "v"):
        t = torch.zeros(B, qc, H, D, dtype=torch.bfloat16)
        for b, inp in enumerate(inputs):
            x = getattr(inp, name)
            t[b, :x.shape[0]] = x
        out.append(t.cuda())
    return out


def _run(config):
    sessions = workloads.session_list(config)
    specs = [s for s, _ in sessions]
    inputs = [workloads.draw_session(s, seed) for s, seed in sessions]
    win = StreamingWindow(specs)
    win.load_window(inputs)
    q, k, v = _chunk_tensors(win, inputs)
    win.step(q, k, v)
    torch.cuda.synchronize()
    win.check_status()
    return specs, inputs, win


@pytest.mark.parametrize("config", [1, 2, 3, 4, 5])
def test_step_matches_oracle(config):
    specs, inputs, win = _run(config)
    o = win.o.cpu()
    lse = win.lse.cpu()
    heads_sel, n_rand = SAMPLING[config]
    worst = (0.0, 0.0)
    for b, (spec, inp) in enumerate(zip(specs, inputs)):
        if heads_sel is None:
            heads, rows = list(range(spec.n_heads)), list(range(spec.chunk_len))
        elif isinstance(heads_sel, int):
            heads, rows = [(7 * b) % spec.n_heads], sample_rows(spec.chunk_len, n_rand, seed=b)
        else:
            heads, rows = heads_sel, sample_rows(spec.chunk_len, n_rand, seed=config)
        ref_o, ref_l = oracle.session_reference(spec, inp, heads=heads, rows=rows)
        for hi, h in enumerate(heads):
            mx, mean = attn_errors(o[b, rows, h], ref_o[:, hi])
            worst = (max(worst[0], mx), max(worst[1], mean))
            assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (config, b, h, mx, mean)
            assert np.all(np.abs(lse[b, h, rows].double().numpy() - ref_l[:, hi]) <= lse_bound(spec, inp, h, rows))
    print(f"\nconfig {config}: max-abs {worst[0]:.3e}  mean-abs {worst[1]:.3e}")


@pytest.mark.parametrize("config", [1, 2, 3, 5])
def test_window_layout_matches_oracle(config):
    """Segment capacities and offsets, the position of every slot and the raw
    K / V bytes of the window equal the oracle's layout: bit-exact for copied
    tokens and positions, within one bf16 ulp for pooled tokens; padding
    stays zero."""
    specs, inputs, win = _run(config)
    assert win.caps == olayout.capacities(specs)
    assert win.offsets == olayout.segment_offsets(olayout.capacities(specs))
    pos = win.pos.cpu().numpy()
    for b, (spec, inp) in enumerate(zip(specs, inputs)):
        segs = oracle.session_kv(spec, inp)
        mask = np.zeros(win.cap_total, bool)
        for seg, off in zip(segs, win.offsets):
            n = seg["k"].shape[0]
            mask[off:off + n] = True
            assert np.array_equal(pos[b, off:off + n], seg["pos"].astype(np.float32)), seg["name"]
            got_k = win.k_raw[b, :, off:off + n].permute(1, 0, 2).cpu()
            got_v = win.v[b, :, off:off + n].permute(1, 0, 2).cpu()
            if seg["name"].startswith("tier"):
                assert ulp_diff_bf16(got_k, seg["k"]).max() <= 1
                assert ulp_diff_bf16(got_v, seg["v"]).max() <= 1
            else:
                assert np.array_equal(got_k.double().numpy(), seg["k"]), seg["name"]
                assert np.array_equal(got_v.double().numpy(), seg["v"]), seg["name"]
        assert not win.v[b, :, torch.from_numpy(~mask).cuda()].any()
        assert not np.any(pos[b, ~mask])
