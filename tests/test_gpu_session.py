"""Whole-step parity on the five workload configs (needs a B200).

The CUDA path runs exactly as the bench runs it (``StreamingWindow``: window
fill with device pooling, then a2 append -> a3 RoPE -> a4 attention); the
oracle recomputes the same step in fp64 from the same seeded inputs.  Full
sizes are checked on sampled (row, head) outputs that include every tile
boundary and the ragged tail; the tiny config and the two streaming chunks
are checked in full (every head, every row)."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import layout as olayout
import workloads
from streaming_video_audio_b200.window import StreamingWindow
from tests.helpers import (ATTN_MAX_ABS, ATTN_MEAN_ABS, LSE_ABS, assert_rope_close, attn_errors, sample_rows,
                           ulp_diff_bf16)

pytestmark = pytest.mark.gpu

# (heads checked per session, random rows per session) for each config:
# None = every head and every row (the oracle needs ~10 s for configs 2 and 3
# on the host cores); an int n = n heads per session, spread over the heads
SAMPLING = {1: (None, None), 2: (None, None), 3: (None, None), 4: ([0, 13, 26, 39], 48), 5: (3, 16)}


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
            heads = sorted({(7 * b + 13 * i) % spec.n_heads for i in range(heads_sel)})
            rows = sample_rows(spec.chunk_len, n_rand, seed=b)
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
    """Segment capacities and offsets, the position of every slot and the
    K / V of the window equal the oracle's layout: bit-exact for copied
    tokens and positions, within one bf16 ulp for pooled tokens; padding
    stays zero.  Keys before RoPE (k_raw) are checked for the history; the
    chunk's keys enter rotated (k_att only), and every segment's rotated
    keys equal the oracle's rotation of its keys at the template positions
    (clock 0, before any slide) within the RoPE tolerance."""
    specs, inputs, win = _run(config)
    assert win.caps == olayout.capacities(specs)
    assert win.offsets == olayout.segment_offsets(olayout.capacities(specs))
    assert float(win.clock.item()) == 0.0
    pos = win.pos.cpu().numpy()
    split, base = tuple(specs[0].rope_split), float(specs[0].rope_base)
    for b, (spec, inp) in enumerate(zip(specs, inputs)):
        segs = oracle.session_kv(spec, inp)
        mask = np.zeros(win.cap_total, bool)
        for seg, off in zip(segs, win.offsets):
            n = seg["k"].shape[0]
            mask[off:off + n] = True
            assert np.array_equal(pos[b, off:off + n], seg["pos"].astype(np.float32)), seg["name"]
            got_v = win.v[b, :, off:off + n].permute(1, 0, 2).cpu()
            rot = win.k_att[b, :, off:off + n].permute(1, 0, 2).cpu()
            if seg["name"] == "chunk":
                # the chunk's keys enter rotated (k_att only)
                assert_rope_close(rot, oracle.rope3d(seg["k"], seg["pos"], split, base), seg["k"])
                assert np.array_equal(got_v.double().numpy(), seg["v"]), seg["name"]
                continue
            got_k = win.k_raw[b, :, off:off + n].permute(1, 0, 2).cpu()
            # rotated once at load, from the window's own bf16 keys
            assert_rope_close(rot, oracle.rope3d(got_k.double().numpy(), seg["pos"], split, base), got_k)
            if seg["name"].startswith("tier"):
                assert ulp_diff_bf16(got_k, seg["k"]).max() <= 1
                assert ulp_diff_bf16(got_v, seg["v"]).max() <= 1
            else:
                assert np.array_equal(got_k.double().numpy(), seg["k"]), seg["name"]
                assert np.array_equal(got_v.double().numpy(), seg["v"]), seg["name"]
        assert not win.v[b, :, torch.from_numpy(~mask).cuda()].any()
        assert not np.any(pos[b, ~mask])


def test_step_with_qk_norm_matches_oracle():
    """The layer with QK normalisation: keys are kept before normalisation,
    pooled, then normalised and rotated in one fused kernel every step."""
    spec = workloads.scaled(workloads.CHUNK_TIERED, n_heads=4, prompt_len=37, context_video_tokens=25 * 1008,
                            chunk_video_tokens=1008 + 300, chunk_audio_tokens=20)
    inp = workloads.draw_session(spec, 7)
    gq = 1.0 + 0.2 * workloads.draw_tensor((128,), seed=8).float()
    gk = 1.0 + 0.2 * workloads.draw_tensor((128,), seed=9).float()
    win = StreamingWindow([spec], qk_norm=(gq, gk, 1e-6))
    win.load_window([inp])
    win.step(inp.q.cuda()[None], inp.k.cuda()[None], inp.v.cuda()[None])
    torch.cuda.synchronize()
    win.check_status()
    rows = sample_rows(spec.chunk_len, 64, seed=3)
    ref_o, _ = oracle.session_reference(spec, inp, rows=rows, qk_norm=(gq.double().numpy(), gk.double().numpy(), 1e-6))
    o = win.o.cpu()
    for h in range(spec.n_heads):
        mx, mean = attn_errors(o[0, rows, h], ref_o[:, h])
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (h, mx, mean)


@pytest.mark.parametrize("config", [2, 3])
def test_prefix_self_and_moving_part_match_oracle(config):
    """Prefix queries (prompt + sink) see only the prefix; recent + chunk
    queries see the whole window with recomputed recent K/V; two denoising
    steps are two banks (batch entries) with their own inputs."""
    spec = workloads.scaled(workloads.CONFIGS[config], n_heads=3)
    seeds = [11, 12]                                # one bank per denoising step
    inputs = [workloads.draw_session(spec, s) for s in seeds]
    movs = [workloads.draw_moving(spec, s) for s in seeds]
    win = StreamingWindow([spec, spec])
    win.load_window(inputs)
    stack = lambda name, src: torch.stack([getattr(x, name) for x in src]).cuda()
    o_pre = win.attend_prefix(stack("prefix_q", movs))
    o_mov = win.step_moving(stack("recent_q", movs), stack("recent_k", movs), stack("recent_v", movs),
                            stack("q", inputs), stack("k", inputs), stack("v", inputs))
    torch.cuda.synchronize()
    win.check_status()
    n_pre = spec.prompt_len + workloads.sink_tokens(spec)
    n_mov = workloads.recent_tokens(spec) + spec.chunk_len
    for b in range(2):
        rows = sample_rows(n_pre, 32, seed=b)
        ref, _ = oracle.prefix_reference(spec, inputs[b], movs[b], rows=rows)
        for h in range(3):
            mx, mean = attn_errors(o_pre[b, rows, h].cpu(), ref[:, h])
            assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, ("prefix", b, h, mx, mean)
        rows = sample_rows(n_mov, 48, seed=10 + b)
        ref, _ = oracle.moving_reference(spec, inputs[b], movs[b], rows=rows)
        for h in range(3):
            mx, mean = attn_errors(o_mov[b, rows, h].cpu(), ref[:, h])
            assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, ("moving", b, h, mx, mean)


def test_host_step_pipeline_matches_device_step():
    """The pipelined host-buffer path returns, for every step, exactly the
    output of the device step on the same inputs."""
    from streaming_video_audio_b200.window import HostStepPipeline
    spec = workloads.scaled(workloads.CHUNK, n_heads=4)
    inp = workloads.draw_session(spec, 4)
    win = StreamingWindow([spec])
    win.load_window([inp])
    chunks = []
    for s in range(3):
        x = workloads.draw_session(spec, 50 + s)
        chunks.append(tuple(getattr(x, n)[None].contiguous() for n in ("q", "k", "v")))
    refs = []
    for q, k, v in chunks:
        refs.append(win.step(q.cuda(), k.cuda(), v.cuda()).cpu().clone())
    pipe = HostStepPipeline(win)
    outs = [torch.empty_like(r).pin_memory() for r in refs]
    for (q, k, v), o in zip(chunks, outs):
        pipe.step(q.pin_memory(), k.pin_memory(), v.pin_memory(), o)
    pipe.synchronize()
    for r, o in zip(refs, outs):
        assert torch.equal(r, o)


def test_host_step_pipeline_with_slides_matches_device_steps():
    """With slide=True the pipeline slides the window by the previous step's
    uploaded chunk before each step: outputs equal the device-side sequence
    advance(previous chunk's video K, V) -> step, bit for bit, over enough
    steps that the two staging sets are each reused while a slide reads the
    other."""
    from streaming_video_audio_b200.window import HostStepPipeline
    spec = workloads.scaled(workloads.CHUNK_TIERED, n_heads=2)
    n = spec.chunk_video_tokens
    inp = workloads.draw_session(spec, 5)
    chunks = [tuple(workloads.draw_tensor((1, spec.chunk_len, 2, 128), seed=70 + 3 * s + j) for j in range(3))
              for s in range(6)]
    win = StreamingWindow([spec])
    win.load_window([inp])
    refs = []
    for s, (q, k, v) in enumerate(chunks):
        if s:
            win.advance(chunks[s - 1][1][:, :n].cuda(), chunks[s - 1][2][:, :n].cuda())
        refs.append(win.step(q.cuda(), k.cuda(), v.cuda()).cpu().clone())
    win2 = StreamingWindow([spec])
    win2.load_window([inp])
    pipe = HostStepPipeline(win2)
    outs = [torch.empty_like(r).pin_memory() for r in refs]
    for (q, k, v), o in zip(chunks, outs):
        pipe.step(q.pin_memory(), k.pin_memory(), v.pin_memory(), o, slide=True)
    pipe.synchronize()
    win2.check_status()
    for r, o in zip(refs, outs):
        assert torch.equal(r, o)


@pytest.mark.parametrize("n_frames", [3, 2])
def test_window_slide_matches_oracle(n_frames):
    """Streaming over successive chunks: after every slide (a1 in streaming
    use: re-pooling at the tier boundaries, the previous chunk's clean frames
    into the recent ring, positions of the new ring state) the step equals
    the oracle's step on the window defined afresh one chunk later.  Chunks
    of 2 frames make the 9- and 3-frame rings wrap inside a slide.

    Window contents per ring, in age order: recent frames bit-exact, tier1
    (pooled once) within one bf16 ulp, tier0 (re-pooled from bf16 tier1
    frames) within the two-rounding bound 2^-9 (max|T2| + |T3|)."""
    ft = workloads.FT
    spec = workloads.scaled(workloads.CHUNK_TIERED, n_heads=3, prompt_len=37, chunk_video_tokens=n_frames * ft)
    H, D, L = spec.n_heads, spec.head_dim, spec.chunk_len
    inp = workloads.draw_session(spec, 21)
    win = StreamingWindow([spec])
    win.load_window([inp])
    win.step(inp.q.cuda()[None], inp.k.cuda()[None], inp.v.cuda()[None])
    n_slides = 13 if n_frames == 3 else 10
    # |T2| never exceeds the largest full-resolution value that ever entered the history
    amax = {"k": max(t.abs().max().item() for t in inp.ctx_k), "v": max(t.abs().max().item() for t in inp.ctx_v)}
    for i in range(n_slides):
        ck, cv = inp.k[:n_frames * ft], inp.v[:n_frames * ft]   # the finished chunk's video K / V
        amax = {"k": max(amax["k"], ck.abs().max().item()), "v": max(amax["v"], cv.abs().max().item())}
        q, k, v = (workloads.draw_tensor((L, H, D), seed=300 + 3 * i + j) for j in range(3))
        win.advance(ck.cuda()[None], cv.cuda()[None])
        win.step(q.cuda()[None], k.cuda()[None], v.cuda()[None])
        inp = oracle.slide_window(spec, inp, ck, cv, q, k, v)
        if i not in (0, 1, 3, n_slides - 2, n_slides - 1):
            continue
        torch.cuda.synchronize()
        win.check_status()
        rows = sample_rows(L, 24, seed=i)
        ref_o, ref_l = oracle.session_reference(spec, inp, rows=rows)
        o, lse = win.o.cpu(), win.lse.cpu()
        for h in range(H):
            mx, mean = attn_errors(o[0, rows, h], ref_o[:, h])
            assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (i, h, mx, mean)
            # the re-pooled tier adds one rounding to its keys: twice the per-score bound
            bound = 2.0 * (lse_bound(spec, inp, h, rows) - LSE_ABS) + LSE_ABS
            assert np.all(np.abs(lse[0, h, rows].double().numpy() - ref_l[:, h]) <= bound), i
        segs = {s["name"]: s for s in oracle.session_kv(spec, inp)}
        pos = win.pos.cpu().numpy()
        for role, r in win.rings.items():
            order = [(win.ring_ptr[role] + j) % r["frames"] for j in range(r["frames"])]
            off, tok = win.seg[role][0], r["tok"]
            slots = np.concatenate([np.arange(off + s * tok, off + (s + 1) * tok) for s in order])
            assert np.array_equal(pos[0, slots], segs[role]["pos"].astype(np.float32)), (i, role)
            idx = torch.from_numpy(slots).cuda()
            for buf, name in ((win.k_raw, "k"), (win.v, "v")):
                got = buf[0][:, idx].permute(1, 0, 2).cpu()
                ref = segs[role][name]
                if role == "recent":
                    assert np.array_equal(got.double().numpy(), ref), (i, role, name)
                elif role == "tier1":
                    assert ulp_diff_bf16(got, ref).max() <= 1, (i, role, name)
                else:
                    err = np.abs(got.double().numpy() - ref)
                    assert np.all(err <= 2.0 ** -9 * (amax[name] + np.abs(ref)) + 1e-12), (i, role, name)


def test_graph_step_matches_eager_steps():
    """The streaming step replayed from CUDA graphs (slide + append + RoPE,
    attention) gives the eager sequence advance -> step bit for bit, over
    more than a full period of ring states (inputs changed in place)."""
    spec = workloads.scaled(workloads.CHUNK_TIERED, n_heads=2)
    n = spec.chunk_video_tokens
    inp = workloads.draw_session(spec, 6)
    chunks = [tuple(workloads.draw_tensor((1, spec.chunk_len, 2, 128), seed=90 + 3 * s + j) for j in range(3))
              for s in range(15)]
    eager = StreamingWindow([spec])
    eager.load_window([inp])
    graphed = StreamingWindow([spec])
    graphed.load_window([inp])
    q, k, v = (torch.zeros(1, spec.chunk_len, 2, 128, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    kc = torch.zeros(1, n, 2, 128, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    for s_, (cq, ck, cv) in enumerate(chunks):
        clean = chunks[s_ - 1] if s_ else chunks[-1]
        eager.advance(clean[1][:, :n].cuda(), clean[2][:, :n].cuda())
        ref = eager.step(cq.cuda(), ck.cuda(), cv.cuda()).cpu()
        for dst, src in ((q, cq), (k, ck), (v, cv), (kc, clean[1][:, :n]), (vc, clean[2][:, :n])):
            dst.copy_(src)
        out = graphed.graph_step(q, k, v, kc, vc).cpu()
        torch.cuda.synchronize()
        assert torch.equal(out, ref), s_
        assert graphed.ring_ptr == eager.ring_ptr
    graphed.check_status()
    assert len(graphed._step_graphs) == eager.period


def test_checkpoint_resume_continues_bit_for_bit():
    """A session saved after four slides (export_state: window buffers, ring
    pointers, position tables) and restored into a fresh window built from
    the same spec continues the stream exactly: the next slide and step give
    the same output and LSE bits as the window that never stopped."""
    spec = workloads.scaled(workloads.CHUNK_TIERED, n_heads=2)
    n = spec.chunk_video_tokens
    inp = workloads.draw_session(spec, 12)
    chunks = [tuple(workloads.draw_tensor((1, spec.chunk_len, 2, 128), seed=500 + 3 * s + j).cuda() for j in range(3))
              for s in range(6)]
    live = StreamingWindow([spec])
    live.load_window([inp])
    live.step(*chunks[0])
    for s_ in range(1, 5):
        live.advance(chunks[s_ - 1][1][:, :n], chunks[s_ - 1][2][:, :n])
        live.step(*chunks[s_])
    state = live.export_state()
    resumed = StreamingWindow([spec])
    resumed.import_state(state)
    for win in (live, resumed):
        win.advance(chunks[4][1][:, :n], chunks[4][2][:, :n])
        win.step(*chunks[5])
    torch.cuda.synchronize()
    live.check_status()
    resumed.check_status()
    assert resumed.ring_ptr == live.ring_ptr
    assert torch.equal(resumed.o, live.o) and torch.equal(resumed.lse, live.lse)
    assert torch.equal(resumed.pos, live.pos)
