"""Kernel-level parity of the CUDA path against the fp64 oracle (needs a B200).

Inputs come from ``workloads`` (seeded draws); expected values only from
``oracle``.  Every call goes through the C ABI (``capi``)."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from streaming_video_audio_b200 import capi
from tests.helpers import ATTN_MAX_ABS, ATTN_MEAN_ABS, LSE_ABS, assert_rope_close, attn_errors, ulp_diff_bf16

pytestmark = pytest.mark.gpu

DEV = "cuda"


# ---------------------------------------------------------------- RoPE (a3)


@pytest.mark.parametrize("D,split,H,N", [(128, (32, 48, 48), 40, 300), (64, (16, 24, 24), 3, 77),
                                         (128, (32, 48, 48), 5, 1),
                                         (128, (32, 48, 48), 72, 33)])   # past 8 head passes: the tail loop
def test_rope_token_major_to_head_major(D, split, H, N):
    B = 2
    x = workloads.draw_tensor((B, N, H, D), seed=1)
    pos = torch.stack([workloads.draw_positions(N, seed=2 + b) for b in range(B)])
    pos[:, :, 0] = torch.round(pos[:, :, 0] * 20) / 20          # mixes integer and fractional t
    y = torch.full((B, H, N + 5, D), 7.0, dtype=torch.bfloat16, device=DEV)
    n_valid = torch.tensor([N, max(1, N - 3)], dtype=torch.int32, device=DEV)
    capi.sr_rope3d_apply(x.to(DEV), y[:, :, :N].permute(0, 2, 1, 3), pos.to(DEV), split, n_valid=n_valid)
    torch.cuda.synchronize()
    for b in range(B):
        nv = int(n_valid[b])
        ref = oracle.rope3d(x[b, :nv], pos[b, :nv].double(), split)        # [nv, H, D]
        got = y[b, :, :nv].permute(1, 0, 2).cpu()
        assert_rope_close(got, ref, x[b, :nv])
        # skipped tokens and padding slots untouched
        assert torch.all(y[b, :, nv:].float().cpu() == 7.0)


def test_rope_zero_position_copy_and_scale():
    D, split, H, N = 128, (32, 48, 48), 4, 130
    x = workloads.draw_tensor((1, N, H, D), seed=3)
    y = torch.empty(1, N, H, D, dtype=torch.bfloat16, device=DEV)
    capi.sr_rope3d_apply(x.to(DEV), y, None, split)
    assert torch.equal(y.cpu(), x)
    capi.sr_rope3d_apply(x.to(DEV), y, None, split, out_scale=0.5)
    assert torch.equal(y.cpu(), (x.float() * 0.5).to(torch.bfloat16))


# ---------------------------------------------------------------- pooling (a1)
@pytest.mark.parametrize("grid,pool,D", [((24, 42), (2, 2), 128), ((24, 42), (4, 4), 128), ((12, 21), (2, 2), 128),
                                         ((5, 7), (4, 4), 64), ((6, 8), (3, 2), 64)])
def test_history_compress(grid, pool, D):
    gh, gw = grid
    ph, pw = pool
    B, F, H = 2, 3, 3
    cells = (-(-gh // ph)) * (-(-gw // pw))
    k = workloads.draw_tensor((B, F, gh * gw, H, D), seed=4)
    v = workloads.draw_tensor((B, F, gh * gw, H, D), seed=5)
    ko = torch.zeros(B, F, cells, H, D, dtype=torch.bfloat16, device=DEV)
    vo = torch.zeros_like(ko)
    frame_t = torch.tensor([[-9.0, -8.0, -7.0], [-3.0, -2.0, -1.0]], device=DEV)
    pos = torch.zeros(B, F * cells, 3, device=DEV)
    slot = torch.full((F * gh * gw,), -1, dtype=torch.int32, device=DEV)
    capi.sr_history_compress(k.to(DEV), v.to(DEV), ko, vo, grid, pool, frame_t=frame_t, pos_out=pos,
                             slot_of_src=slot)
    torch.cuda.synchronize()
    for b in range(B):
        for src, out in ((k, ko), (v, vo)):
            ref = oracle.pool(src[b].reshape(F, gh, gw, H, D), ph, pw).reshape(F, cells, H, D)
            assert ulp_diff_bf16(out[b].cpu(), ref).max() <= 1
    # positions and the slot map are index arithmetic: bit-exact
    from oracle import layout
    cell_pos = np.array([(mr, mc) for (_, _, _, _, mr, mc) in layout.pooled_cells(gh, gw, ph, pw)])
    exp = np.zeros((B, F * cells, 3), np.float32)
    for b in range(B):
        for f in range(F):
            exp[b, f * cells:(f + 1) * cells, 0] = frame_t[b, f].item()
            exp[b, f * cells:(f + 1) * cells, 1:] = cell_pos
    assert np.array_equal(pos.cpu().numpy(), exp)
    exp_slot = np.empty(F * gh * gw, np.int32)
    for f in range(F):
        for j, (r0, r1, c0, c1, _, _) in enumerate(layout.pooled_cells(gh, gw, ph, pw)):
            for r in range(r0, r1):
                for c in range(c0, c1):
                    exp_slot[f * gh * gw + r * gw + c] = f * cells + j
    assert np.array_equal(slot.cpu().numpy(), exp_slot)


def test_history_compress_two_stage_matches_direct():
    """T2 -> T3 re-pooling on the device vs direct 4x4 pooling of the
    full-resolution frames (equal in exact arithmetic on a 24x42 grid).  The
    bound follows from the two roundings: each T2 value is off by at most
    2^-9 of its magnitude, their mean by at most 2^-9 max|T2|, and the final
    rounding adds 2^-9 |T3|."""
    H, D = 4, 128
    k = workloads.draw_tensor((1, 2, 1008, H, D), seed=6)
    t2 = torch.zeros(1, 2, 252, H, D, dtype=torch.bfloat16, device=DEV)
    t3 = torch.zeros(1, 2, 66, H, D, dtype=torch.bfloat16, device=DEV)
    capi.sr_history_compress(k.to(DEV), None, t2, None, (24, 42), (2, 2))
    capi.sr_history_compress(t2, None, t3, None, (12, 21), (2, 2))
    ref = oracle.pool(k[0].reshape(2, 24, 42, H, D), 4, 4).reshape(2, 66, H, D)
    t2max = np.abs(oracle.pool(k[0].reshape(2, 24, 42, H, D), 2, 2)).max()
    err = np.abs(t3[0].cpu().double().numpy() - ref)
    assert np.all(err <= 2.0 ** -9 * (t2max + np.abs(ref)) + 1e-12)


# ---------------------------------------------------------------- append (a2)
def test_kv_append_exact_and_in_place():
    B, H, D, cap, N = 2, 5, 128, 512, 200
    kb = torch.zeros(B, H, cap, D, dtype=torch.bfloat16, device=DEV)
    vb = torch.zeros_like(kb)
    pb = torch.zeros(B, cap, 3, device=DEV)
    ks = workloads.draw_tensor((B, N, H, D), seed=7)
    vs = workloads.draw_tensor((B, N, H, D), seed=8)
    ps = torch.stack([workloads.draw_positions(N, seed=9), workloads.draw_positions(N, seed=10)])
    nv = torch.tensor([N, 150], dtype=torch.int32, device=DEV)
    capi.sr_kv_append(kb, vb, pb, 100, ks.to(DEV), vs.to(DEV), ps.to(DEV), n_valid=nv)
    torch.cuda.synchronize()
    for b, n in enumerate((N, 150)):
        assert torch.equal(kb[b, :, 100:100 + n].cpu(), ks[b, :n].permute(1, 0, 2))
        assert torch.equal(vb[b, :, 100:100 + n].cpu(), vs[b, :n].permute(1, 0, 2))
        assert torch.equal(pb[b, 100:100 + n].cpu(), ps[b, :n])
        assert not kb[b, :, :100].any() and not kb[b, :, 100 + n:].any()
        assert not pb[b, 100 + n:].any()


@pytest.mark.parametrize("with_raw", [True, False])
def test_kv_append_with_fused_rotation(with_raw):
    """The cache write and the RoPE in one pass: K lands rotated in k_rot at
    its position plus the stream clock (t_origin), optionally also unrotated
    in k_buf (bit-exact copy), V is copied bit-exactly; slots outside
    [dst, dst + n_valid) stay untouched."""
    B, H, D, cap, N, dst = 2, 40, 128, 512, 200, 128
    split = (32, 48, 48)
    kb = torch.zeros(B, H, cap, D, dtype=torch.bfloat16, device=DEV)
    kr = torch.zeros_like(kb)
    vb = torch.zeros_like(kb)
    ks = workloads.draw_tensor((B, N, H, D), seed=17)
    vs = workloads.draw_tensor((B, N, H, D), seed=18)
    ps = torch.stack([workloads.draw_positions(N, seed=19), workloads.draw_positions(N, seed=20)])
    clock = torch.tensor([1234.0], dtype=torch.float64, device=DEV)
    nv = torch.tensor([N, 150], dtype=torch.int32, device=DEV)
    rot = capi.RopeOut(kr, ps.to(DEV), split, t_origin=clock)
    capi.sr_kv_append(kb if with_raw else None, vb, None, dst, ks.to(DEV), vs.to(DEV), None, n_valid=nv, rot=rot)
    torch.cuda.synchronize()
    for b, n in enumerate((N, 150)):
        shifted = ps[b, :n].double().numpy() + np.array([1234.0, 0.0, 0.0])
        ref = oracle.rope3d(ks[b, :n], shifted, split)
        assert_rope_close(kr[b, :, dst:dst + n].permute(1, 0, 2).cpu(), ref, ks[b, :n])
        assert torch.equal(vb[b, :, dst:dst + n].cpu(), vs[b, :n].permute(1, 0, 2))
        if with_raw:
            assert torch.equal(kb[b, :, dst:dst + n].cpu(), ks[b, :n].permute(1, 0, 2))
        else:
            assert not kb.any()
        for t in (kr, vb):
            assert not t[b, :, :dst].any() and not t[b, :, dst + n:].any()


def test_history_compress_with_fused_rotation():
    """Pooling with the pooled key rotated on its way into the tier: k_rot
    equals the RoPE (at the given cell positions plus the clock) of the
    pooled bf16 key k_out holds."""
    gh, gw, ph, pw, B, F, H, D = 24, 42, 2, 2, 1, 3, 40, 128
    split = (32, 48, 48)
    cells = 12 * 21
    k = workloads.draw_tensor((B, F, gh * gw, H, D), seed=24)
    v = workloads.draw_tensor((B, F, gh * gw, H, D), seed=25)
    ko = torch.zeros(B, F, cells, H, D, dtype=torch.bfloat16, device=DEV)
    vo, kr = torch.zeros_like(ko), torch.zeros_like(ko)
    rpos = torch.stack([workloads.draw_positions(F * cells, seed=26)]).to(DEV)
    clock = torch.tensor([-57.0], dtype=torch.float64, device=DEV)
    capi.sr_history_compress(k.to(DEV), v.to(DEV), ko, vo, (gh, gw), (ph, pw),
                             rot=capi.RopeOut(kr, rpos, split, t_origin=clock))
    torch.cuda.synchronize()
    pooled = ko[0].reshape(F * cells, H, D).cpu()
    ref = oracle.rope3d(pooled, rpos[0].double().cpu().numpy() + np.array([-57.0, 0.0, 0.0]), split)
    assert_rope_close(kr[0].reshape(F * cells, H, D).cpu(), ref, pooled)
    ref_v = oracle.pool(v[0].reshape(F, gh, gw, H, D), ph, pw).reshape(F, cells, H, D)
    assert ulp_diff_bf16(vo[0].cpu(), ref_v).max() <= 1


def test_rope_t_origin_and_stream_clock():
    """t_origin adds the stream clock to every t (formed in fp64): the result
    matches the oracle's rotation at the shifted positions; the clock kernel
    adds exactly."""
    B, N, H, D = 1, 64, 8, 128
    split = (32, 48, 48)
    x = workloads.draw_tensor((B, N, H, D), seed=33)
    pos = workloads.draw_positions(N, seed=34)[None]
    clock = torch.zeros(1, dtype=torch.float64, device=DEV)
    for _ in range(7):
        capi.sr_stream_clock_advance(clock, 3.0)
    capi.sr_stream_clock_advance(clock, 0.5)
    torch.cuda.synchronize()
    assert float(clock.item()) == 21.5
    y = torch.zeros(B, H, N, D, dtype=torch.bfloat16, device=DEV)
    capi.sr_rope3d_apply(x.to(DEV), y.permute(0, 2, 1, 3), pos.to(DEV), split, t_origin=clock)
    torch.cuda.synchronize()
    ref = oracle.rope3d(x[0], pos[0].double().numpy() + np.array([21.5, 0.0, 0.0]), split)
    assert_rope_close(y[0].permute(1, 0, 2).cpu(), ref, x[0])


# ---------------------------------------------------------------- attention (a4)
def _draw_case(D, H, caps, lens, q_len, seed, perturb_padding=False):
    """Seeded bf16 q/k/v in the kernel's layout (padding optionally filled with
    large finite garbage)."""
    B = len(lens)
    C = sum(caps)
    q_cap = max(q_len)
    q = workloads.draw_tensor((B, H, q_cap, D), seed=seed)
    k = workloads.draw_tensor((B, H, C, D), seed=seed + 1, scale=0.7)
    v = workloads.draw_tensor((B, H, C, D), seed=seed + 2)
    if perturb_padding:
        rng = np.random.default_rng(seed + 3)
        for b in range(B):
            off = 0
            for cap, n in zip(caps, lens[b]):
                pad = slice(off + n, off + cap)
                for t in (k, v):
                    shape = t[b, :, pad].shape
                    t[b, :, pad] = torch.from_numpy(rng.uniform(-60, 60, shape).astype(np.float32)).to(torch.bfloat16)
                off += cap
    return q, k, v


def _run_attention(q, k, v, caps, lens, q_len, use_workspace=True):
    B, H, q_cap, D = q.shape
    o = torch.full((B, q_cap, H, D), 3.0, dtype=torch.bfloat16, device=DEV)
    lse = torch.zeros(B, H, q_cap, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    nbytes = capi.sr_chunk_attention_workspace_bytes(B, H, D, q_cap)
    ws = torch.full((max(nbytes, 16),), 0xAB, dtype=torch.uint8, device=DEV) if use_workspace and nbytes else None
    capi.sr_chunk_attention_fwd(q.to(DEV).contiguous(), k.to(DEV).contiguous(), v.to(DEV).contiguous(), o, lse,
                                caps, torch.tensor(lens, dtype=torch.int32, device=DEV),
                                torch.tensor(q_len, dtype=torch.int32, device=DEV), 1 / math.sqrt(D), status,
                                workspace=ws)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o.cpu(), lse.cpu()


def _attention_case(D, H, caps, lens, q_len, seed, perturb_padding=False):
    q, k, v = _draw_case(D, H, caps, lens, q_len, seed, perturb_padding)
    o, lse = _run_attention(q, k, v, caps, lens, q_len)
    return q, k, v, o, lse


def _valid_kv(k, v, b, h, caps, lens_b):
    idx, off = [], 0
    for cap, n in zip(caps, lens_b):
        idx += list(range(off, off + n))
        off += cap
    return k[b, h, idx], v[b, h, idx]


@pytest.mark.parametrize("D,H,caps,lens,q_len", [
    (128, 2, [256, 512, 384], [[200, 300, 333]], [333]),
    (64, 1, [128, 128, 128], [[16, 96, 100]], [100]),
    (128, 3, [128, 1024, 256], [[1, 1000, 129], [128, 7, 256], [0, 513, 255]], [129, 256, 255]),
    (64, 2, [256, 256], [[256, 256], [1, 0]], [200, 1]),
    (128, 2, [128, 256], [[128, 200], [64, 9]], [256, 0]),      # a session without queries
    # the most segments a window may have, empty ones between full and ragged ones
    (128, 2, [128, 256, 128, 384, 128, 128, 256, 128], [[100, 0, 128, 300, 0, 1, 256, 77]], [300]),
    (64, 3, [256, 128, 128, 128, 128, 128, 128, 256], [[0, 0, 5, 128, 0, 64, 0, 255]], [130]),
])
def test_attention_matches_oracle(D, H, caps, lens, q_len):
    q, k, v, o, lse = _attention_case(D, H, caps, lens, q_len, seed=20)
    for b in range(len(lens)):
        if q_len[b] == 0:
            assert torch.all(o[b] == 3.0)      # nothing written
            continue
        for h in range(H):
            kk, vv = _valid_kv(k, v, b, h, caps, lens[b])
            ro, rl = oracle.attention(q[b, h, :q_len[b]], kk, vv, 1 / math.sqrt(D))
            mx, mean = attn_errors(o[b, :q_len[b], h], ro)
            assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (b, h, mx, mean)
            assert np.abs(lse[b, h, :q_len[b]].double().numpy() - rl).max() <= LSE_ABS
        # rows beyond q_len untouched
        assert torch.all(o[b, q_len[b]:] == 3.0)


def test_attention_ignores_padding_and_other_sessions():
    """Finite garbage in padded slots and the presence of other sessions in
    the batch change no output bit."""
    D, H, caps = 128, 2, [128, 384, 256]
    lens = [[100, 300, 200], [128, 257, 129]]
    args = (D, H, caps, lens, [200, 129])
    _, _, _, o1, l1 = _attention_case(*args, seed=30)
    _, _, _, o2, l2 = _attention_case(*args, seed=30, perturb_padding=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    q, k, v = _draw_case(*args, seed=30)
    o3, l3 = _run_attention(q[:1], k[:1], v[:1], caps, lens[:1], [200])
    assert torch.equal(o3[0, :200], o1[0, :200]) and torch.equal(l3[0, :, :200], l1[0, :, :200])


def test_attention_all_segments_empty_writes_zeros():
    D, H, caps = 64, 1, [128, 128]
    _, _, _, o, lse = _attention_case(D, H, caps, [[0, 0]], [5], seed=40)
    assert torch.all(o[0, :5] == 0) and torch.all(torch.isinf(lse[0, 0, :5]))


def test_attention_split_schedule_matches_whole_units():
    """With a workspace the last partial wave is split along the KV tiles and
    merged in fp32; without one every unit runs whole.  Both are checked
    against the oracle and against each other."""
    D, H, caps = 128, 5, [256, 1024, 384]
    lens = [[256, 1000, 300]]
    q_len = [700]
    nbytes = capi.sr_chunk_attention_workspace_bytes(1, H, D, 700)
    assert nbytes > 0   # 5 heads x 3 query blocks < one wave: split is active
    q, k, v = _draw_case(D, H, caps, lens, q_len, seed=50)
    o_split, l_split = _run_attention(q, k, v, caps, lens, q_len, use_workspace=True)
    o_whole, l_whole = _run_attention(q, k, v, caps, lens, q_len, use_workspace=False)
    assert float((o_split[0, :700].float() - o_whole[0, :700].float()).abs().max()) <= 2 ** -7
    assert float((l_split[0, :, :700] - l_whole[0, :, :700]).abs().max()) <= 1e-4
    for h in range(H):
        kk, vv = _valid_kv(k, v, 0, h, caps, lens[0])
        ro, rl = oracle.attention(q[0, h, :700], kk, vv, 1 / math.sqrt(D))
        for o_ in (o_split, o_whole):
            mx, mean = attn_errors(o_[0, :700, h], ro)
            assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS


def test_attention_repeated_launches_deterministic():
    """Many launches of ragged, few-tile work (split parts of one or two tiles,
    empty parts, empty segments): no pipeline wait may give up and every
    launch must produce the same bits."""
    D, H, caps = 128, 3, [128, 1024, 256]
    lens = [[1, 1000, 129], [128, 7, 256], [0, 513, 255]]
    q_len = [129, 256, 255]
    q, k, v = _draw_case(D, H, caps, lens, q_len, seed=60)
    o0, l0 = _run_attention(q, k, v, caps, lens, q_len)
    for _ in range(40):
        o, l = _run_attention(q, k, v, caps, lens, q_len)
        assert torch.equal(o, o0) and torch.equal(l, l0)
    for _ in range(10):
        o, l = _run_attention(q, k, v, caps, lens, q_len, use_workspace=False)
        assert torch.equal(o[0, :129], _run_attention(q, k, v, caps, lens, q_len, use_workspace=False)[0][0, :129])


@pytest.mark.parametrize("use_workspace", [True, False])
def test_attention_q_len_past_q_cap_writes_inside_buffers(use_workspace):
    """A device q_len larger than q_cap (the host cannot see it) is clamped in
    the kernels: rows [0, q_cap) are computed as for q_len = q_cap and guard
    memory after o and lse keeps its sentinel.  q_cap = 300 is not a multiple
    of the 256-row query block, so the last block reaches past the buffer."""
    D, H, caps, lens, q_cap = 128, 2, [256, 512], [[256, 400]], 300
    q, k, v = _draw_case(D, H, caps, lens, [q_cap], seed=45)
    guard = 300
    o_full = torch.full((q_cap + guard, H, D), 7.0, dtype=torch.bfloat16, device=DEV)
    lse_full = torch.full((H * q_cap + 2 * guard,), 7.0, dtype=torch.float32, device=DEV)
    o, lse = o_full[:q_cap].view(1, q_cap, H, D), lse_full[:H * q_cap].view(1, H, q_cap)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    nbytes = capi.sr_chunk_attention_workspace_bytes(1, H, D, q_cap)
    assert nbytes > 0
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV) if use_workspace else None
    capi.sr_chunk_attention_fwd(q.to(DEV).contiguous(), k.to(DEV).contiguous(), v.to(DEV).contiguous(), o, lse,
                                caps, torch.tensor(lens, dtype=torch.int32, device=DEV),
                                torch.tensor([q_cap + 100], dtype=torch.int32, device=DEV), 1 / math.sqrt(D),
                                status, workspace=ws)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.all(o_full[q_cap:] == 7.0) and torch.all(lse_full[H * q_cap:] == 7.0)
    for h in range(H):
        kk, vv = _valid_kv(k, v, 0, h, caps, lens[0])
        ro, rl = oracle.attention(q[0, h], kk, vv, 1 / math.sqrt(D))
        mx, mean = attn_errors(o[0, :, h].cpu(), ro)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (h, mx, mean)
        assert np.abs(lse[0, h].double().cpu().numpy() - rl).max() <= LSE_ABS


@pytest.mark.parametrize("D", [128, 64])
def test_attention_wait_runs_out_reports_timeout_and_context_survives(D):
    """Failure detection without a GPU fault: with the load of K tile 1
    withheld (the library's test hook) and a 2 ms wait limit, the pipeline
    wait for that tile runs out; the launch writes SR_ERR_DEVICE_TIMEOUT into
    the status word, waits for its own loads and MMAs in flight, releases its
    tensor memory and returns.  The context stays usable: the next normal
    launch matches the oracle."""
    H, caps, lens, q_len = 2, [256, 512], [[200, 400]], [300]
    q, k, v = _draw_case(D, H, caps, lens, q_len, seed=47)
    qd, kd, vd = (t.to(DEV).contiguous() for t in (q, k, v))
    kl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    ql = torch.tensor(q_len, dtype=torch.int32, device=DEV)
    o = torch.zeros(1, 300, H, D, dtype=torch.bfloat16, device=DEV)
    lse = torch.zeros(1, H, 300, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    capi.sr_set_wait_limit_ns(2_000_000)
    capi.sr_set_withheld_kv_tile(1)
    try:
        # whole units (no workspace): every work item walks all 6 KV tiles
        capi.sr_chunk_attention_fwd(qd, kd, vd, o, lse, caps, kl, ql, 1 / math.sqrt(D), status, workspace=None)
        torch.cuda.synchronize()
    finally:
        capi.sr_set_withheld_kv_tile(-1)
        capi.sr_set_wait_limit_ns(0)
    assert int(status.item()) == capi.SR_ERR_DEVICE_TIMEOUT
    o2, l2 = _run_attention(q, k, v, caps, lens, q_len)
    for h in range(H):
        kk, vv = _valid_kv(k, v, 0, h, caps, lens[0])
        ro, rl = oracle.attention(q[0, h, :300], kk, vv, 1 / math.sqrt(D))
        mx, mean = attn_errors(o2[0, :300, h], ro)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (h, mx, mean)


# ---------------------------------------------------------------- QK-norm + RoPE (fused)
@pytest.mark.parametrize("D,split,H,N", [(128, (32, 48, 48), 40, 200), (64, (16, 24, 24), 5, 33),
                                         (128, (32, 48, 48), 56, 3), (128, (32, 48, 48), 64, 17)])
def test_qknorm_rope_matches_oracle(D, split, H, N):
    B = 2
    x = workloads.draw_tensor((B, N, H, D), seed=90, scale=3.0)
    gamma = (1.0 + 0.1 * workloads.draw_tensor((D,), seed=91).float()).contiguous()
    pos = torch.stack([workloads.draw_positions(N, seed=92 + b) for b in range(B)])
    y = torch.zeros(B, H, N, D, dtype=torch.bfloat16, device=DEV)
    y_raw = torch.zeros(B, N, H, D, dtype=torch.bfloat16, device=DEV)
    capi.sr_qknorm_rope3d_apply(x.to(DEV), y.permute(0, 2, 1, 3), gamma.to(DEV), 1e-6, pos.to(DEV), split,
                                y_raw=y_raw)
    torch.cuda.synchronize()
    for b in range(B):
        u = oracle.rms_norm(x[b], gamma.double(), 1e-6)                  # [N, H, D]
        assert ulp_diff_bf16(y_raw[b].cpu(), u).max() <= 1
        ref = oracle.rope3d(u, pos[b].double(), split)
        assert_rope_close(y[b].permute(1, 0, 2).cpu(), ref, torch.from_numpy(u))


# ---------------------------------------------------------------- gather / scatter (window partition)
def _gather_case(B, S, T, seed):
    """idx [B, S]: distinct source tokens with -1 holes (slot order shuffled)."""
    rng = np.random.default_rng(seed)
    idx = np.full((B, S), -1, dtype=np.int32)
    perm = rng.permutation(T)
    k = 0
    for b in range(B):
        n = min(S, T - k, int(rng.integers(S // 2, S + 1)))
        slots = np.sort(rng.choice(S, size=n, replace=False))
        idx[b, slots] = perm[k:k + n]
        k += n
    return idx


@pytest.mark.parametrize("D,H", [(128, 4), (128, 12), (64, 3)])
def test_gather_and_scatter_tokens_exact(D, H):
    B, S, T = 5, 40, 170
    src = workloads.draw_tensor((T, H, D), seed=140)
    pos = workloads.draw_positions(T, seed=141)
    idx = _gather_case(B, S, T, seed=142)
    dst = torch.full((B, S, H, D), 3.0, dtype=torch.bfloat16, device=DEV)
    dpos = torch.full((B, S, 3), 5.0, device=DEV)
    capi.sr_gather_tokens(dst, src.to(DEV), torch.from_numpy(idx).to(DEV), src_pos=pos.to(DEV), dst_pos=dpos)
    back = torch.full((T, H, D), 9.0, dtype=torch.bfloat16, device=DEV)
    capi.sr_scatter_tokens(back, dst, torch.from_numpy(idx).to(DEV))
    torch.cuda.synchronize()
    d, p, bk = dst.cpu(), dpos.cpu(), back.cpu()
    for b in range(B):
        for s_ in range(S):
            t = int(idx[b, s_])
            if t >= 0:
                assert torch.equal(d[b, s_], src[t]) and torch.equal(p[b, s_], pos[t])
            else:
                assert not d[b, s_].any() and not p[b, s_].any()
    hit = np.zeros(T, bool)
    hit[idx[idx >= 0]] = True
    assert torch.equal(bk[torch.from_numpy(hit)], src[torch.from_numpy(hit)])
    assert bool((bk[torch.from_numpy(~hit)] == 9.0).all())


@pytest.mark.parametrize("D,split,H", [(128, (32, 48, 48), 4), (128, (32, 48, 48), 10), (64, (16, 24, 24), 2)])
def test_gather_rope3d_tokens_matches_oracle(D, split, H):
    """The gathered rows rotated by their source token's position: within the
    RoPE tolerance of the fp64 oracle; holes are zero."""
    B, S, T = 4, 48, 150
    src = workloads.draw_tensor((T, H, D), seed=150)
    pos = workloads.draw_positions(T, seed=151)
    pos[:, 0] = torch.round(pos[:, 0] * 20) / 20
    idx = _gather_case(B, S, T, seed=152)
    dst = torch.full((B, H, S, D), 3.0, dtype=torch.bfloat16, device=DEV)   # head-major, as the ring
    capi.sr_gather_rope3d_tokens(dst.permute(0, 2, 1, 3), src.to(DEV), torch.from_numpy(idx).to(DEV), pos.to(DEV),
                                 split)
    torch.cuda.synchronize()
    got = dst.permute(0, 2, 1, 3).cpu()
    sel = idx >= 0
    rows = idx[sel]
    ref = oracle.rope3d(src[rows], pos[rows].double(), split)
    assert_rope_close(got[torch.from_numpy(sel)], ref, src[rows])
    assert not got[torch.from_numpy(~sel)].any()


# ---------------------------------------------------------------- windowed attention (causal VAE decoder)
@pytest.mark.parametrize("D,split,shift", [(64, (16, 24, 24), 0), (64, (16, 24, 24), 8), (128, (32, 48, 48), 8)])
def test_ring_window_attention_matches_oracle(D, split, shift):
    """Four calls of 2 latent frames through a 6-frame ring (empty, half-full,
    full, wrapped) on a grid whose edge windows are partial."""
    from oracle import vae_window
    from streaming_video_audio_b200.vae_window import RingWindowAttention
    gh, gw, H, calls = 20, 36, 2, 4
    T = gh * gw
    F = 2 * calls
    q = workloads.draw_tensor((F, T, H, D), seed=100)
    k = workloads.draw_tensor((F, T, H, D), seed=101)
    v = workloads.draw_tensor((F, T, H, D), seed=102)
    layer = RingWindowAttention((gh, gw), H, D, split, shift=shift)
    t0 = 57                                     # stream clock of frame 0
    for c in range(calls):
        fr = slice(2 * c, 2 * c + 2)
        o = layer(q[fr].reshape(2 * T, H, D).cuda(), k[fr].reshape(2 * T, H, D).cuda(),
                  v[fr].reshape(2 * T, H, D).cuda(), t0=t0 + 2 * c)
        torch.cuda.synchronize()
        assert int(layer.status.item()) == 0
        ref = vae_window.window_attention_reference(q[:2 * c + 2], k[:2 * c + 2], v[:2 * c + 2], (gh, gw), t0=t0,
                                                    call_frames=2, history=4, split=split, shift=shift)
        mx, mean = attn_errors(o.cpu(), ref)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (c, mx, mean)


def test_ring_window_attention_graph_replay_equals_eager_calls():
    """Eight calls (every ring state twice) replayed from CUDA graphs give the
    eager calls' outputs bit for bit; inputs change in place between calls."""
    from streaming_video_audio_b200.vae_window import RingWindowAttention
    gh, gw, H, D, T = 20, 36, 2, 128, 20 * 36
    frames = [tuple(workloads.draw_tensor((2 * T, H, D), seed=130 + 3 * c + j) for j in range(3)) for c in range(8)]
    eager = RingWindowAttention((gh, gw), H, D, (32, 48, 48), shift=8)
    ref = [eager(*(t.cuda() for t in fr), t0=5 + 2 * c).cpu() for c, fr in enumerate(frames)]
    layer = RingWindowAttention((gh, gw), H, D, (32, 48, 48), shift=8)
    q, k, v = (torch.zeros(2 * T, H, D, dtype=torch.bfloat16, device=DEV) for _ in range(3))
    out = torch.zeros(2 * T, H, D, dtype=torch.bfloat16, device=DEV)
    for c, fr in enumerate(frames):
        for dst, src in zip((q, k, v), fr):
            dst.copy_(src)
        layer.graphed(q, k, v, t0=5 + 2 * c, out=out)
        torch.cuda.synchronize()
        assert int(layer.status.item()) == 0
        assert torch.equal(out.cpu(), ref[c]), c
    assert len(layer.graphs) == 5     # (first slot, phase): (0,0) (2,1) (4,2) (0,2) (2,2)


def test_ring_window_attention_is_causal_and_clock_invariant():
    """Changing a later call's frames leaves earlier outputs bit-identical, and
    starting the stream clock elsewhere changes nothing but rounding."""
    from streaming_video_audio_b200.vae_window import RingWindowAttention
    gh, gw, H, D, T = 20, 36, 2, 64, 20 * 36
    q = workloads.draw_tensor((6, T, H, D), seed=110)
    k = workloads.draw_tensor((6, T, H, D), seed=111)
    v = workloads.draw_tensor((6, T, H, D), seed=112)

    def run(qq, kk, vv, t0):
        layer = RingWindowAttention((gh, gw), H, D, (16, 24, 24), shift=8)
        outs = []
        for c in range(3):
            fr = slice(2 * c, 2 * c + 2)
            outs.append(layer(qq[fr].reshape(2 * T, H, D).cuda(), kk[fr].reshape(2 * T, H, D).cuda(),
                              vv[fr].reshape(2 * T, H, D).cuda(), t0=t0 + 2 * c).cpu())
        return outs

    a = run(q, k, v, 0)
    k2, v2 = k.clone(), v.clone()
    k2[4:] = workloads.draw_tensor((2, T, H, D), seed=113)
    v2[4:] = workloads.draw_tensor((2, T, H, D), seed=114)
    b = run(q, k2, v2, 0)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and not torch.equal(a[2], b[2])
    c = run(q, k, v, 1000)
    for x, y in zip(a, c):
        assert float((x.float() - y.float()).abs().max()) <= 2e-2
