"""The allocation-free attention entry point (needs a B200).

sr_chunk_attention_fwd_noalloc serves callers that cannot allocate device
memory when they run the attention -- a plugin handed only its input and
output buffers, a real-time loop that must not call cudaMalloc, an
application whose memory belongs to its own allocator.  It takes its split-KV
scratch from a static device array inside the library instead of a
caller-provided workspace.  This test calls it through the C ABI twice in a
row, on two different problems that both use the scratch, and compares each
result with the regular entry point given an ordinary workspace.  It lives in
its own file, collected last, and needs nothing from the other tests.
"""
import math

import pytest
import torch

import workloads
from streaming_video_audio_b200 import capi
from tests.helpers import ATTN_MAX_ABS, ATTN_MEAN_ABS, attn_errors

pytestmark = pytest.mark.gpu

DEV = "cuda"

# (head_dim, heads, segment capacities, valid lengths per session, query lengths, seed)
CASES = [
    (128, 5, [256, 1024, 384], [[256, 1000, 300]], [700], 70),
    (128, 3, [128, 512, 256], [[100, 512, 256], [7, 300, 129]], [256, 129], 80),
]


def _inputs(D, H, caps, lens, q_len, seed):
    B, C, qc = len(lens), sum(caps), max(q_len)
    q = workloads.draw_tensor((B, H, qc, D), seed=seed).to(DEV)
    k = workloads.draw_tensor((B, H, C, D), seed=seed + 1, scale=0.7).to(DEV)
    v = workloads.draw_tensor((B, H, C, D), seed=seed + 2).to(DEV)
    return q, k, v


def _outputs(B, H, qc, D):
    return (torch.full((B, qc, H, D), 5.0, dtype=torch.bfloat16, device=DEV),
            torch.zeros(B, H, qc, device=DEV), torch.zeros(1, dtype=torch.int32, device=DEV))


def test_noalloc_attention_matches_regular_entry_point_twice_in_a_row():
    torch.cuda.set_device(0)
    prepared = []
    for D, H, caps, lens, q_len, seed in CASES:
        B, qc = len(lens), max(q_len)
        need = capi.sr_chunk_attention_workspace_bytes(B, H, D, qc)
        assert 0 < need <= capi.SR_NOALLOC_SCRATCH_BYTES   # the static scratch is really used
        q, k, v = _inputs(D, H, caps, lens, q_len, seed)
        kv_len = torch.tensor(lens, dtype=torch.int32, device=DEV)
        ql = torch.tensor(q_len, dtype=torch.int32, device=DEV)
        scale = 1.0 / math.sqrt(D)
        o_ref, l_ref, s_ref = _outputs(B, H, qc, D)
        ws = torch.empty(need, dtype=torch.uint8, device=DEV)
        capi.sr_chunk_attention_fwd(q, k, v, o_ref, l_ref, caps, kv_len, ql, scale, s_ref, workspace=ws)
        prepared.append((q, k, v, caps, kv_len, ql, scale, lens, q_len, o_ref, l_ref, s_ref))
    torch.cuda.synchronize()
    # two allocation-free calls back to back; the second finds the first's
    # data still in the shared scratch
    results = []
    for q, k, v, caps, kv_len, ql, scale, lens, q_len, *_ in prepared:
        B, H, qc, D = q.shape
        o_na, l_na, s_na = _outputs(B, H, qc, D)
        capi.sr_chunk_attention_fwd_noalloc(q, k, v, o_na, l_na, caps, kv_len, ql, scale, s_na)
        results.append((o_na, l_na, s_na))
    torch.cuda.synchronize()
    for (q, k, v, caps, kv_len, ql, scale, lens, q_len, o_ref, l_ref, s_ref), (o_na, l_na, s_na) in zip(prepared, results):
        assert int(s_ref.item()) == 0 and int(s_na.item()) == 0
        H = q.shape[1]
        for b, n in enumerate(q_len):
            for h in range(H):
                mx, mean = attn_errors(o_na[b, :n, h].cpu(), o_ref[b, :n, h].double().cpu().numpy())
                assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (b, h, mx, mean)
            assert float((l_na[b, :, :n] - l_ref[b, :, :n]).abs().max()) <= 1e-3
            assert torch.all(o_na[b, n:] == 5.0)   # rows past the query length untouched
