"""Pins for the oracle's attention and whole-step composition (CPU only)."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def test_matches_torch_sdpa_fp64():
    q, k, v = _rand((70, 64), 1), _rand((300, 64), 2), _rand((300, 64), 3)
    o, lse = oracle.attention(q, k, v, 1 / 8)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])[0].numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    s = torch.from_numpy(q) @ torch.from_numpy(k).T / 8
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=1).numpy(), rtol=0, atol=1e-12)


def test_brute_force_unshifted_on_tiny_config():
    """Pure-Python O(N^2) loop with un-shifted exp and exactly rounded sums
    (math.fsum) on the tiny config's raw chunk-over-window tensors."""
    sp = workloads.TINY
    inp = workloads.draw_session(sp, 0)
    q = inp.q[:, 0].double().numpy()
    k = torch.cat([inp.prompt_k] + inp.ctx_k + [inp.k])[:, 0].double().numpy()
    v = torch.cat([inp.prompt_v] + inp.ctx_v + [inp.v])[:, 0].double().numpy()
    rows = list(range(0, 100, 7)) + [99]
    o, lse = oracle.attention(q, k, v, 1 / math.sqrt(64), rows=rows)
    for t, i in enumerate(rows):
        w = [math.exp(math.fsum(q[i, d] * k[j, d] for d in range(64)) / 8.0) for j in range(k.shape[0])]
        den = math.fsum(w)
        for d in range(0, 64, 9):
            num = math.fsum(w[j] * v[j, d] for j in range(k.shape[0]))
            assert abs(num / den - o[t, d]) <= 1e-12
        assert abs(math.log(den) - lse[t]) <= 1e-12


def test_rows_sum_to_one_and_nonnegative():
    nk = 48
    q, k = _rand((40, 64), 4, 2.0), _rand((nk, 64), 5, 2.0)
    v = np.zeros((nk, 64))
    v[np.arange(nk), np.arange(nk)] = 1.0          # o row = the probability row
    o, _ = oracle.attention(q, k, v, 0.125)
    assert np.all(o >= 0)
    np.testing.assert_allclose(o.sum(axis=1), 1.0, rtol=0, atol=1e-12)


def test_equal_keys_give_mean_value():
    q = _rand((10, 64), 6)
    k = np.tile(_rand((1, 64), 7), (33, 1))
    v = _rand((33, 64), 8)
    o, lse = oracle.attention(q, k, v, 0.125)
    np.testing.assert_allclose(o, np.tile(v.mean(axis=0), (10, 1)), atol=1e-13)


def test_single_key_gives_its_value():
    q, k, v = _rand((5, 128), 9), _rand((1, 128), 10), _rand((1, 128), 11)
    o, lse = oracle.attention(q, k, v, 1 / math.sqrt(128))
    np.testing.assert_array_equal(o, np.tile(v, (5, 1)))
    np.testing.assert_allclose(lse, (q @ k.T)[:, 0] / math.sqrt(128), atol=1e-13)


def test_key_permutation_invariance():
    q, k, v = _rand((20, 64), 12), _rand((90, 64), 13), _rand((90, 64), 14)
    perm = np.random.default_rng(15).permutation(90)
    o1, l1 = oracle.attention(q, k, v, 0.125)
    o2, l2 = oracle.attention(q, k[perm], v[perm], 0.125)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def test_segment_split_lse_combination():
    """Attention over [A | B | C] equals the LSE-weighted mix of per-segment results."""
    q = _rand((16, 64), 16)
    ks = [_rand((n, 64), 17 + i) for i, n in enumerate((16, 96, 100))]
    vs = [_rand((n, 64), 27 + i) for i, n in enumerate((16, 96, 100))]
    o, lse = oracle.attention(q, np.concatenate(ks), np.concatenate(vs), 0.125)
    parts = [oracle.attention(q, kk, vv, 0.125) for kk, vv in zip(ks, vs)]
    L = np.stack([p[1] for p in parts], 1)
    w = np.exp(L - lse[:, None])
    np.testing.assert_allclose(w.sum(1), 1.0, atol=1e-12)
    mix = sum(w[:, i:i + 1] * parts[i][0] for i in range(3))
    np.testing.assert_allclose(mix, o, atol=1e-12)


def test_session_reference_shift_invariance():
    """Moving the window clock and the h, w origins of every rotated token
    leaves O unchanged: only position differences enter q.k after RoPE.
    (The prompt is unrotated, so the check uses a window without prompt.)"""
    from oracle import layout
    sp = workloads.scaled(workloads.TINY, prompt_len=0)
    inp = workloads.draw_session(sp, 3)
    o_ref, l_ref = oracle.session_reference(sp, inp)
    segs = oracle.session_kv(sp, inp)
    k = np.concatenate([s["k"] for s in segs])
    v = np.concatenate([s["v"] for s in segs])
    for shift in ([100.0, 3.0, -5.0], [0.15, 0.0, 0.0], [1000.0, 0.0, 0.0]):
        sh = np.asarray([shift])
        kr = oracle.rope3d(k, np.concatenate([s["pos"] for s in segs]) + sh, sp.rope_split)
        qr = oracle.rope3d(inp.q.double().numpy(), np.asarray(layout.chunk_positions(sp)) + sh, sp.rope_split)
        o, l = oracle.attention(qr[:, 0], kr[:, 0], v[:, 0], 0.125)
        np.testing.assert_allclose(o, o_ref[:, 0], atol=1e-10)
        np.testing.assert_allclose(l, l_ref[:, 0], atol=1e-10)


def test_session_reference_matches_sdpa_composition():
    """The whole step equals torch SDPA (fp64, CPU) over the rotated window,
    for a case with several segments, tiers and audio tokens."""
    sp = workloads.scaled(workloads.CHUNK_TIERED, n_heads=2, head_dim=64, rope_split=(16, 24, 24),
                          prompt_len=9, chunk_video_tokens=1008 + 17, chunk_audio_tokens=5)
    inp = workloads.draw_session(sp, 21)
    rows = [0, 1, 500, 1024, 1025, 1029]
    o, lse = oracle.session_reference(sp, inp, rows=rows)
    segs = oracle.session_kv(sp, inp)
    k = np.concatenate([s["k"] for s in segs])
    v = np.concatenate([s["v"] for s in segs])
    p = np.concatenate([s["pos"] for s in segs])
    from oracle import layout
    kr = torch.from_numpy(oracle.rope3d(k, p, sp.rope_split)).permute(1, 0, 2)
    qr = torch.from_numpy(oracle.rope3d(inp.q.double().numpy(), np.asarray(layout.chunk_positions(sp)),
                                        sp.rope_split)).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(qr, kr, torch.from_numpy(v).permute(1, 0, 2))
    np.testing.assert_allclose(o, ref.permute(1, 0, 2).numpy()[rows], atol=1e-12)


def test_prefix_and_moving_references_reduce_to_plain_attention():
    """The prefix-self attention equals plain attention of the prefix queries
    over [prompt | sink] keys; the moving-part attention of the chunk rows
    equals the whole-step reference once the recent frames' K/V are swapped
    for the recomputed ones; without a prefix-only mask the prefix rows would
    differ (the mask matters)."""
    sp = workloads.scaled(workloads.TINY, prompt_len=5)
    inp = workloads.draw_session(sp, 2)
    mov = workloads.draw_moving(sp, 2)
    o_pre, l_pre = oracle.prefix_reference(sp, inp, mov)
    segs = {s["name"]: s for s in oracle.session_kv(sp, inp)}
    k = np.concatenate([segs["prompt"]["k"], segs["sink"]["k"]])[:, 0]
    v = np.concatenate([segs["prompt"]["v"], segs["sink"]["v"]])[:, 0]
    p = np.concatenate([segs["prompt"]["pos"], segs["sink"]["pos"]])
    kr = torch.from_numpy(oracle.rope3d(k, p, sp.rope_split))[None]
    qr = torch.from_numpy(oracle.rope3d(mov.prefix_q[:, 0].double().numpy(), p, sp.rope_split))[None]
    ref = torch.nn.functional.scaled_dot_product_attention(qr, kr, torch.from_numpy(v)[None])[0].numpy()
    np.testing.assert_allclose(o_pre[:, 0], ref, atol=1e-12)
    # moving part: the chunk rows see the recomputed recent frames
    o_mov, _ = oracle.moving_reference(sp, inp, mov)
    assert o_mov.shape[0] == workloads.recent_tokens(sp) + sp.chunk_len
    inp2 = workloads.SessionInputs(inp.prompt_k, inp.prompt_v, inp.ctx_k[:1] + [mov.recent_k], inp.ctx_v[:1] + [mov.recent_v],
                                   inp.q, inp.k, inp.v)
    o_step, _ = oracle.session_reference(sp, inp2)
    np.testing.assert_allclose(o_mov[workloads.recent_tokens(sp):], o_step, atol=1e-12)
