"""The window slide on the host (CPU only): the ring pointer logic and the
position tables of ``StreamingWindow`` against the oracle's definition of the
window one chunk later (``oracle.slide_window`` + ``oracle.session_kv``).

The device kernels are replaced by an fp64 executor of the planned calls (the
oracle's own pooling), so the test pins what is pooled where and which
position each slot takes, over a full period of ring states and past it."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from streaming_video_audio_b200.window import StreamingWindow

FT = workloads.FT
SPEC = workloads.scaled(workloads.CHUNK_TIERED, n_heads=1, head_dim=128, prompt_len=8, chunk_audio_tokens=4)


def _clean(i, n=3):
    return (workloads.draw_tensor((n * FT, 1, 128), seed=500 + 2 * i),
            workloads.draw_tensor((n * FT, 1, 128), seed=501 + 2 * i))


def _long_video(n_frames, seed):
    return [workloads.draw_tensor((FT, 1, 128), seed=seed + f) for f in range(n_frames)]


def test_slide_window_oracle_equals_later_window_of_one_video():
    """Pin of the oracle's slide: a window over frames [s, s+24) of one video
    slid by the next 3 frames is the window over [s+3, s+27) (sink kept)."""
    video_k, video_v = _long_video(40, 1000), _long_video(40, 2000)
    base = workloads.draw_session(SPEC, 0)

    def window_at(s):
        return type(base)(base.prompt_k, base.prompt_v, [video_k[0]] + video_k[1 + s:25 + s],
                          [video_v[0]] + video_v[1 + s:25 + s], base.q, base.k, base.v)

    w = window_at(2)
    slid = oracle.slide_window(SPEC, w, torch.cat(video_k[27:30]), torch.cat(video_v[27:30]), w.q, w.k, w.v)
    ref = window_at(5)
    assert len(slid.ctx_k) == 25
    for a, b in zip(slid.ctx_k + slid.ctx_v, ref.ctx_k + ref.ctx_v):
        assert torch.equal(a, b)


def _window_cpu(n=3):
    win = StreamingWindow([SPEC], device="cpu")
    win._ring_setup(n)
    return win


def test_ring_state_zero_positions_are_the_loaded_template():
    win = _window_cpu()
    pos = win.ring_positions(win.ring_ptr)
    segs = {s["name"]: s for s in oracle.session_kv(SPEC, workloads.draw_session(SPEC, 0))}
    for role in win.rings:
        off = win.seg[role][0]
        n = segs[role]["pos"].shape[0]
        assert np.array_equal(pos[off:off + n], segs[role]["pos"].astype(np.float32)), role
    assert win.period == 12    # tier0: 12 / 3, tier1: 9 / 3, recent: 3 / 3


@pytest.mark.parametrize("n", [3, 2, 1])
def test_slide_plan_matches_oracle_over_a_period(n):
    """n = 3 (a chunk of 3 frames) keeps every pointer on a multiple of 3;
    n = 2 and 1 make the 9- and 3-frame rings wrap inside a slide."""
    win = _window_cpu(n)
    inp = workloads.draw_session(SPEC, 0)
    segs = {s["name"]: s for s in oracle.session_kv(SPEC, inp)}
    state = {}
    for role, r in win.rings.items():
        state[role] = segs[role]["k"].reshape(r["frames"], r["tok"], -1).copy()
    ptr = dict(win.ring_ptr)
    wraps = 0
    seen = set()
    for i in range(win.period + 2):
        seen.add(tuple(ptr.values()))
        ck, cv = _clean(i, n)
        ops, ptr_next = win.slide_ops(ptr)
        wraps += sum(1 for op in ops if op[0] == "pool" and op[5] < n)
        for op in ops:
            if op[0] == "pool":
                _, src, fs, dst, fd, m, (gh, gw), (ph, pw) = op
                x = state[src][fs:fs + m].reshape(m, gh, gw, -1)
                state[dst][fd:fd + m] = oracle.pool(x, ph, pw).reshape(m, -1, x.shape[-1])
            else:
                _, fr, fc, m = op
                state["recent"][fr:fr + m] = ck.double().numpy().reshape(n, FT, -1)[fc:fc + m]
        ptr = ptr_next
        inp = oracle.slide_window(SPEC, inp, ck, cv, inp.q, inp.k, inp.v)
        segs = {s["name"]: s for s in oracle.session_kv(SPEC, inp)}
        pos = win.ring_positions(ptr)
        for role, r in win.rings.items():
            order = [(ptr[role] + j) % r["frames"] for j in range(r["frames"])]
            ref_k = segs[role]["k"].reshape(r["frames"], r["tok"], -1)
            np.testing.assert_allclose(state[role][order], ref_k, rtol=0, atol=1e-12, err_msg=f"{role} slide {i}")
            off = win.seg[role][0]
            got_pos = np.concatenate([pos[off + s * r["tok"]:off + (s + 1) * r["tok"]] for s in order])
            assert np.array_equal(got_pos, segs[role]["pos"].astype(np.float32)), (role, i)
    assert len(seen) == win.period == {3: 12, 2: 18, 1: 36}[n]
    assert (wraps > 0) == (n == 2)


def test_slide_rejects_inputs_it_cannot_place():
    win = StreamingWindow([SPEC], device="cpu")
    with pytest.raises(ValueError):
        win._ring_setup(4)          # more frames than the 3-frame recent ring
    spec = workloads.scaled(workloads.CHUNK, context_video_tokens=4 * FT - 10)
    with pytest.raises(ValueError):
        StreamingWindow([spec], device="cpu")._ring_setup(1)     # partial history frame


@pytest.mark.parametrize("config", [1, 2, 3, 4, 5])
def test_window_layout_and_chunk_positions_match_oracle_on_host(config):
    """Segment capacities, offsets and the chunk's position template of the
    product's window (host side) against the oracle's own layout code."""
    from oracle import layout as olayout
    specs = [s for s, _ in workloads.session_list(config)]
    win = StreamingWindow(specs, device="cpu")
    assert win.caps == olayout.capacities(specs)
    assert win.offsets == olayout.segment_offsets(olayout.capacities(specs))
    for b, spec in enumerate(specs):
        ref = np.asarray(olayout.chunk_positions(spec), dtype=np.float32)
        assert np.array_equal(win.q_pos[b, :spec.chunk_len].numpy(), ref)
        assert not win.q_pos[b, spec.chunk_len:].any()
        assert [int(x) for x in win.lengths[b]] == olayout.segment_lengths(spec)
