"""The multi-GPU host logic on CPU: two gloo ranks (spawned processes).

Each rank runs its own sessions (different seeds, same shapes, so per-rank
work is fixed: weak scaling); the bench takes the max of every timing over
ranks and divides the work of all ranks by it.  No data-path collective."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads
        sess = bench.rank_sessions(3, rank)
        seeds = [seed for _, seed in sess]
        specs = [sp for sp, _ in sess]
        # fake per-rank timings: rank r is (r + 1) times slower
        local = [10.0 * (rank + 1), 20.0 * (rank + 1), 5.0 * (rank + 1)]
        agg = bench.aggregate(local, flops_per_step=1e12, steps=4, world=world, group=dist.group.WORLD)
        # the draws of different ranks differ; their shapes do not
        x = workloads.draw_session(workloads.scaled(specs[0], n_heads=1, head_dim=64, rope_split=(16, 24, 24),
                                                    context_video_tokens=1008, tiers=(), prompt_len=4,
                                                    chunk_video_tokens=16, chunk_audio_tokens=0), seeds[0])
        gathered = [torch.zeros_like(x.q.float()) for _ in range(world)]
        dist.all_gather(gathered, x.q.float())
        out[rank] = {"seeds": seeds, "agg": agg, "distinct": not torch.equal(gathered[0], gathered[1]),
                     "shapes": [tuple(g.shape) for g in gathered]}
    finally:
        dist.destroy_process_group()


def test_two_rank_sharding_and_max_over_ranks_timing():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as manager:
        out = manager.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=240)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0]["seeds"] == [0] and res[1]["seeds"] == [1000]
    for r in range(world):
        agg = res[r]["agg"]
        assert agg["total_ms"] == 20.0 and agg["e2e_ms"] == 40.0 and agg["attn_ms"] == 10.0   # max over ranks
        assert abs(agg["value"] - 2 * 1e12 * 4 / 0.020 / 1e12) < 1e-9                            # all ranks' work
    assert res[0]["distinct"] and res[0]["shapes"][0] == res[0]["shapes"][1]
