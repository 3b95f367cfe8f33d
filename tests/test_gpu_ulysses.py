"""Ulysses sequence parallelism on the GPU (needs a B200).

Several ranks are emulated in one process on one device: each rank's window
holds its heads, the two all-to-alls are done by copies between the rank
objects, and no kernel waits on another (the host runs the phases in
order).  The assembled output is compared with the oracle's all-head step.
A one-rank NCCL group runs the real ``step`` with its collectives and must
reproduce the unsharded window bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from streaming_video_audio_b200.ulysses import (UlyssesAttention, exchange_back_in_process,
                                                exchange_in_process)
from streaming_video_audio_b200.window import StreamingWindow
from tests.helpers import ATTN_MAX_ABS, ATTN_MEAN_ABS, attn_errors, sample_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 4, 8])
def test_emulated_ranks_match_oracle(world):
    spec = workloads.scaled(workloads.CHUNK_TIERED, n_heads=8, prompt_len=100)
    inp = workloads.draw_session(spec, 31)
    ranks = [UlyssesAttention(spec, r, world) for r in range(world)]
    for ua in ranks:
        ua.load_window(inp)
    outs = []
    for r, ua in enumerate(ranks):
        lo, hi = ua.plan.tokens_of(r)
        ua.pack(inp.q[lo:hi].cuda(), inp.k[lo:hi].cuda(), inp.v[lo:hi].cuda())
    exchange_in_process(ranks)
    for ua in ranks:
        ua.attend()
    exchange_back_in_process(ranks)
    for ua in ranks:
        outs.append(ua.unpack())
    torch.cuda.synchronize()
    for ua in ranks:
        ua.win.check_status()
    o = torch.cat(outs).cpu()
    assert o.shape == (spec.chunk_len, spec.n_heads, spec.head_dim)
    rows = sample_rows(spec.chunk_len, 48, seed=world)
    ref, _ = oracle.session_reference(spec, inp, rows=rows)
    for h in range(spec.n_heads):
        mx, mean = attn_errors(o[rows, h], ref[:, h])
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (world, h, mx, mean)


def test_single_rank_nccl_step_equals_unsharded_window():
    import torch.distributed as dist
    spec = workloads.scaled(workloads.CHUNK, n_heads=4)
    inp = workloads.draw_session(spec, 32)
    win = StreamingWindow([spec])
    win.load_window([inp])
    ref = win.step(inp.q.cuda()[None], inp.k.cuda()[None], inp.v.cuda()[None])[0].cpu()
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1, device_id=torch.device("cuda:0"))
    try:
        ua = UlyssesAttention(spec, 0, 1, group=dist.group.WORLD)
        ua.load_window(inp)
        o = ua.step(inp.q.cuda(), inp.k.cuda(), inp.v.cuda())
        torch.cuda.synchronize()
        ua.win.check_status()
        assert torch.equal(o.cpu(), ref)
    finally:
        dist.destroy_process_group()
