"""Ulysses head re-partition on CPU: the partition arithmetic, and the whole
exchange (pack -> all-to-all -> attention of the local heads -> all-to-all
-> unpack) over real gloo process groups of 2 and 4 spawned ranks.

The local attention is the fp64 oracle on the rank's heads (a test stand-in
for the head-sharded window), so the assembled output must equal the
oracle's all-head result bit for bit after bf16 rounding: heads are
independent, and every byte that crosses the exchange is checked."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads
from streaming_video_audio_b200.ulysses import UlyssesPlan

SPEC = workloads.scaled(workloads.TINY, n_heads=4, chunk_audio_tokens=5)   # 96 video + 5 audio = 101 tokens


def test_plan_partitions_tokens_and_heads():
    for L, H, N in [(101, 4, 2), (101, 4, 4), (3044, 40, 8), (3044, 40, 5), (7, 8, 8), (1, 2, 2)]:
        p = UlyssesPlan(L, H, N)
        toks = [p.tokens_of(r) for r in range(N)]
        assert toks[0][0] == 0 and toks[-1][1] == L
        assert all(a[1] == b[0] for a, b in zip(toks, toks[1:]))               # contiguous, no overlap
        assert all(hi - lo <= p.slice_tokens for lo, hi in toks)
        assert p.slice_tokens * N >= L > p.slice_tokens * (N - 1) or L < N
        heads = [p.heads_of(r) for r in range(N)]
        assert sorted(h for lo, hi in heads for h in range(lo, hi)) == list(range(H))
    with pytest.raises(ValueError):
        UlyssesPlan(101, 4, 3)


class OracleWindow:
    """Stand-in for the head-sharded window: the oracle's step on the
    received chunk for the local heads, rounded to bf16."""

    def __init__(self, spec):
        self.spec = spec

    def load_window(self, inputs):
        x = inputs[0]
        self.inp = workloads.SessionInputs(x.prompt_k, x.prompt_v, list(x.ctx_k), list(x.ctx_v), x.q, x.k, x.v)

    def step(self, q, k, v, out):
        import oracle
        self.seen = tuple(t[0].clone() for t in (q, k, v))
        i = self.inp
        o, _ = oracle.session_reference(self.spec, workloads.SessionInputs(i.prompt_k, i.prompt_v, i.ctx_k, i.ctx_v,
                                                                           q[0], k[0], v[0]))
        out[0].copy_(torch.from_numpy(o).to(torch.bfloat16))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import dataclasses
    import datetime
    import oracle
    from streaming_video_audio_b200.ulysses import UlyssesAttention
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = workloads.draw_session(SPEC, 3)
        plan = UlyssesPlan(SPEC.chunk_len, SPEC.n_heads, world)
        local = dataclasses.replace(SPEC, n_heads=plan.local_heads)
        ua = UlyssesAttention(SPEC, rank, world, group=dist.group.WORLD, device="cpu", window=OracleWindow(local))
        ua.load_window(inp)
        lo, hi = plan.tokens_of(rank)
        o = ua.step(inp.q[lo:hi], inp.k[lo:hi], inp.v[lo:hi])
        h0, h1 = plan.heads_of(rank)
        seen = ua.win.seen
        ref, _ = oracle.session_reference(SPEC, inp, rows=list(range(lo, hi)))
        out[rank] = {
            "recv_exact": all(torch.equal(s, getattr(inp, n)[:, h0:h1]) for s, n in zip(seen, ("q", "k", "v"))),
            "out_exact": torch.equal(o, torch.from_numpy(ref).to(torch.bfloat16)),
            "rows": (lo, hi), "shape": tuple(o.shape),
        }
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_exchange_over_gloo(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as manager:
        out = manager.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
            assert p.exitcode == 0
        res = dict(out)
    assert sorted(res) == list(range(world))
    for r in range(world):
        assert res[r]["recv_exact"], r
        assert res[r]["out_exact"], r
        assert res[r]["shape"][1:] == (SPEC.n_heads, SPEC.head_dim)
    assert res[world - 1]["rows"][1] == SPEC.chunk_len
