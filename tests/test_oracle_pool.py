"""Pins for the oracle's history-tier pooling and its window layout (CPU only)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import layout
import workloads


def _torch_avg_pool(x, ph, pw):
    """Library reference: torch avg_pool2d, ceil mode, padding excluded from
    the count.  x: [F, Gh, Gw, C] float64."""
    t = torch.from_numpy(np.ascontiguousarray(x.transpose(0, 3, 1, 2)))
    y = torch.nn.functional.avg_pool2d(t, (ph, pw), stride=(ph, pw), ceil_mode=True,
                                       count_include_pad=False)
    return y.numpy().transpose(0, 2, 3, 1)


@pytest.mark.parametrize("grid,pool", [((5, 7), (2, 2)), ((5, 7), (4, 4)), ((24, 42), (2, 2)),
                                       ((24, 42), (4, 4)), ((12, 21), (2, 2)), ((6, 8), (3, 2))])
def test_pool_matches_torch_avg_pool(grid, pool):
    x = np.random.default_rng(1).standard_normal((3,) + grid + (5,))
    np.testing.assert_allclose(oracle.pool(x, *pool), _torch_avg_pool(x, *pool), rtol=0, atol=1e-14)


def test_pool_brute_force_tiny():
    Gh, Gw, ph, pw = 5, 7, 4, 4
    x = np.random.default_rng(2).standard_normal((1, Gh, Gw, 1))
    y = oracle.pool(x, ph, pw)
    assert y.shape == (1, 2, 2, 1)
    # cells by hand: rows {0..3},{4}; cols {0..3},{4..6}
    np.testing.assert_allclose(y[0, 0, 0, 0], x[0, 0:4, 0:4, 0].mean(), atol=1e-15)
    np.testing.assert_allclose(y[0, 0, 1, 0], x[0, 0:4, 4:7, 0].sum() / 12.0, atol=1e-15)
    np.testing.assert_allclose(y[0, 1, 0, 0], x[0, 4, 0:4, 0].sum() / 4.0, atol=1e-15)
    np.testing.assert_allclose(y[0, 1, 1, 0], x[0, 4, 4:7, 0].sum() / 3.0, atol=1e-15)


def test_pool_constant_and_mass():
    x = np.full((2, 24, 42, 3), 1.75)
    assert np.all(oracle.pool(x, 4, 4) == 1.75)
    x = np.random.default_rng(3).standard_normal((2, 24, 42, 3))
    y = oracle.pool(x, 4, 4)
    counts = np.array([[(r1 - r0) * (c1 - c0) for (r0, r1, c0, c1, _, _) in layout.pooled_cells(24, 42, 4, 4)]])
    mass = (y.reshape(2, -1, 3) * counts.reshape(1, -1, 1)).sum(axis=1)
    np.testing.assert_allclose(mass, x.sum(axis=(1, 2)), rtol=1e-13)


def test_two_stage_equals_direct_on_divisible_grid():
    """24x42 -> 2x2 -> 2x2 equals 4x4 (ceil) directly: T2 cells are all full."""
    x = np.random.default_rng(4).standard_normal((2, 24, 42, 4))
    np.testing.assert_allclose(oracle.pool(oracle.pool(x, 2, 2), 2, 2), oracle.pool(x, 4, 4), atol=1e-14)


def test_pooled_cell_centroids_match_avg_pool_of_coordinates():
    for (Gh, Gw, ph, pw) in [(24, 42, 4, 4), (24, 42, 2, 2), (5, 7, 4, 4)]:
        rr, cc = np.meshgrid(np.arange(Gh, dtype=float), np.arange(Gw, dtype=float), indexing="ij")
        ref = _torch_avg_pool(np.stack([rr, cc], -1)[None], ph, pw)[0].reshape(-1, 2)
        got = np.array([(mr, mc) for (_, _, _, _, mr, mc) in layout.pooled_cells(Gh, Gw, ph, pw)])
        assert np.array_equal(got, ref)


def test_latent_geometry_from_pages(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "latent_geometry.json")))
    s = g["vae_spatial_compression"] * g["dit_patch_thw"][1]
    assert g["frame_width_px"] // s == workloads.GRID_W_FULL == 42
    assert g["frame_height_px"] // s == workloads.GRID_H_FULL == 24
    assert g["audio_sample_rate_hz"] / g["audio_hop"] == workloads.AUDIO_RATE == 40.0
    assert g["video_fps"] / g["vae_temporal_compression"] == workloads.LATENT_FPS == 6.0
    assert workloads.CHUNK.head_dim == g["head_dim"]


def test_segment_lengths_and_capacities():
    # tiered chunk: sink 1008, 12 frames x (6 x 11) cells, 9 frames x (12 x 21), 3 x 1008, 3 x 1008 + 20
    sp = workloads.CHUNK_TIERED
    assert layout.segment_names(sp) == ["prompt", "sink", "tier0", "tier1", "recent", "chunk"]
    assert layout.segment_lengths(sp) == [256, 1008, 12 * 66, 9 * 252, 3024, 3044]
    assert layout.capacities([sp]) == [256, 1024, 896, 2304, 3072, 3072]
    assert layout.segment_offsets(layout.capacities([sp])) == [0, 256, 1280, 2176, 4480, 7552]
    sp = workloads.CHUNK
    assert layout.segment_lengths(sp) == [256, 1008, 3024, 3044]
    sp = workloads.CLIP
    assert layout.segment_names(sp) == ["prompt", "chunk"]
    assert layout.segment_lengths(sp) == [256, 30440]
    sp = workloads.TINY
    assert layout.segment_lengths(sp) == [16, 48, 48, 100]


def test_positions():
    sp = workloads.CHUNK
    pos = layout.chunk_positions(sp)
    assert len(pos) == 3044
    assert pos[0] == (0.0, 0.0, 0.0) and pos[1] == (0.0, 0.0, 1.0) and pos[42] == (0.0, 1.0, 0.0)
    assert pos[3023] == (2.0, 23.0, 41.0)
    assert pos[3024] == (0.0, 0.0, 0.0)
    # audio i at i * 6 / 40 latent frames: token 20 would sit 0.5 s = 3 latent frames later
    np.testing.assert_allclose([p[0] for p in pos[3024:]], np.arange(20) * 0.15, rtol=0, atol=1e-15)
    plan = layout.context_plan(sp)
    assert [p[0] for p in plan] == [-4.0, -3.0, -2.0, -1.0]
    assert [p[1] for p in plan] == ["sink", "recent", "recent", "recent"]
    plan = layout.context_plan(workloads.CHUNK_TIERED)
    assert plan[0][:2] == (-25.0, "sink")
    assert [p[1] for p in plan[1:13]] == ["tier0"] * 12 and plan[1][0] == -24.0 and plan[12][0] == -13.0
    assert [p[1] for p in plan[13:22]] == ["tier1"] * 9 and plan[21][0] == -4.0
    assert [p[1] for p in plan[22:]] == ["recent"] * 3


def test_session_kv_places_input_tokens():
    sp = workloads.scaled(workloads.CHUNK_TIERED, n_heads=2, head_dim=64, rope_split=(16, 24, 24),
                          prompt_len=7, chunk_video_tokens=2 * 1008 + 5, chunk_audio_tokens=3)
    inp = workloads.draw_session(sp, 11)
    segs = oracle.session_kv(sp, inp)
    by = {s["name"]: s for s in segs}
    assert np.array_equal(by["prompt"]["k"], inp.prompt_k.double().numpy())
    assert np.array_equal(by["sink"]["v"], inp.ctx_v[0].double().numpy())
    assert np.array_equal(by["recent"]["k"], torch.cat(inp.ctx_k[22:]).double().numpy())
    assert np.array_equal(by["chunk"]["v"], inp.v.double().numpy())
    f = np.stack([t.double().numpy() for t in inp.ctx_k[1:13]]).reshape(12, 24, 42, -1)
    ref = _torch_avg_pool(f, 4, 4).reshape(12 * 66, 2, 64)
    np.testing.assert_allclose(by["tier0"]["k"], ref, atol=1e-14)
    assert by["chunk"]["pos"][2 * 1008 + 4].tolist() == [2.0, 0.0, 4.0]
    assert by["tier1"]["pos"][0].tolist() == [-12.0, 0.5, 0.5]
    assert by["tier0"]["pos"][65].tolist() == [-24.0, 21.5, 40.5]


def test_window_reference_reduces_to_full_attention_when_one_window_covers_the_grid():
    """A grid smaller than one window with no shift: every token of the
    history range is in the single window, so the reference is plain
    attention of the current frames over all kept frames."""
    from oracle import vae_window
    F, gh, gw, H, D = 5, 6, 7, 1, 64
    q = workloads.draw_tensor((F, gh * gw, H, D), seed=1)
    k = workloads.draw_tensor((F, gh * gw, H, D), seed=2)
    v = workloads.draw_tensor((F, gh * gw, H, D), seed=3)
    o = vae_window.window_attention_reference(q, k, v, (gh, gw), t0=10, call_frames=2, history=2,
                                              split=(16, 24, 24))
    kept = list(range(1, 5))                      # frames 3, 4 current + 2 of history
    rr, cc = np.divmod(np.arange(gh * gw), gw)
    pos = lambda fs: np.concatenate([np.stack([np.full(gh * gw, 10 + f), rr, cc], 1) for f in fs]).astype(float)
    kr = oracle.rope3d(k[kept, :, 0].reshape(-1, D), pos(kept), (16, 24, 24))
    qr = oracle.rope3d(q[[3, 4], :, 0].reshape(-1, D), pos([3, 4]), (16, 24, 24))
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(qr)[None], torch.from_numpy(kr)[None],
                                                           v[kept, :, 0].reshape(-1, D).double()[None])[0]
    np.testing.assert_allclose(o[:, 0], ref.numpy(), atol=1e-12)


def test_window_membership_partitions_the_grid():
    from oracle import vae_window
    for shift in (0, 8):
        seen = {}
        for r in range(20):
            for c in range(36):
                seen.setdefault(vae_window.window_of(r, c, 16, shift), []).append((r, c))
        assert sum(len(x) for x in seen.values()) == 20 * 36
        assert all(len(x) <= 256 for x in seen.values())
        assert len(seen) == (-(-(20 + shift) // 16)) * (-(-(36 + shift) // 16))


def test_window_reference_sees_only_its_window_and_its_history():
    """Pins of the ring-window reference: (1) frames older than the history
    leave the current output unchanged, one frame inside it does not;
    (2) a token changed in one window leaves every other window's output
    unchanged and changes its own; (3) the shift moves the window borders."""
    from oracle import vae_window
    F, gh, gw, H, D = 5, 20, 20, 1, 64
    kw = dict(grid_hw=(gh, gw), t0=3, call_frames=2, history=2, split=(16, 24, 24))
    q = workloads.draw_tensor((F, gh * gw, H, D), seed=21)
    k = workloads.draw_tensor((F, gh * gw, H, D), seed=22)
    v = workloads.draw_tensor((F, gh * gw, H, D), seed=23)
    base = vae_window.window_attention_reference(q, k, v, **kw)
    # (1) frame 0 is outside the 2-frame history of the call on frames 3, 4; frame 1 is inside
    k2, v2 = k.clone(), v.clone()
    k2[0] += 1.0
    v2[0] -= 2.0
    assert np.array_equal(vae_window.window_attention_reference(q, k2, v2, **kw), base)
    v3 = v.clone()
    v3[1] += 1.0
    assert not np.allclose(vae_window.window_attention_reference(q, k, v3, **kw), base)
    # (2) change the value of token (row 2, col 3) of frame 2: window (0, 0) only (no shift)
    v4 = v.clone()
    v4[2, 2 * gw + 3] += 5.0
    out = vae_window.window_attention_reference(q, k, v4, **kw)
    rows = np.arange(2 * gh * gw) % (gh * gw)
    in_w00 = ((rows // gw) < 16) & ((rows % gw) < 16)
    assert np.array_equal(out[~in_w00], base[~in_w00])
    assert not np.allclose(out[in_w00], base[in_w00])
    # (3) with shift 8 the same token's window is the corner one: rows and cols [0, 8)
    kw8 = dict(kw, shift=8)
    base8 = vae_window.window_attention_reference(q, k, v, **kw8)
    out8 = vae_window.window_attention_reference(q, k, v4, **kw8)
    in_w = ((rows // gw) < 8) & ((rows % gw) < 8)
    assert np.array_equal(out8[~in_w], base8[~in_w])
    assert not np.allclose(out8[in_w], base8[in_w])
