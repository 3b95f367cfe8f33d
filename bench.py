"""Benchmark of the chunk-streaming joint video+audio attention step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config {2,3,4,5}] [--impl {sr,reference}]

A step is one pass of the whole hot path on one batch of synthetic inputs
resident in HBM: the window slide of the tiered configs (a1: the frames that
cross a tier boundary are pooled into the older tier and the previous chunk's
clean frames become the recent ones), KV append of the chunk (a2), RoPE of
the chunk queries and of every window key (a3) and the fused chunk attention
(a4).  Default workload: the tiered streaming chunk (config 3), the one
config on which all four steps run.

Printed: ONE JSON line (rank 0) with attention TFLOP/s of the whole job
(algorithmic FLOPs 4*Lq*Lkv*D per head over valid tokens only, summed over
ranks, divided by the max-over-ranks time of K steps), ms per step, the
attention kernel's roofline (CUDA events on the launch stream), clocks
sampled during the timed region, an end-to-end figure through
``StreamingWindow.step_from_host`` (pinned host buffers, copies inside the
timed region) and the fp64 oracle timed on a bounded sample on the host.

Multi-GPU (torchrun): every rank runs its own sessions (seed offset by
rank); there is no data-path collective (weak scaling).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

CONFIG_DESC = {
    1: "tiny: 1 head x 64, chunk 2x6x8 video + 4 audio over 16 prompt + 2 context frames",
    2: "chunk: one streaming chunk at 1344x768 (3 latent frames x 1008 + 20 audio) over 256 prompt + "
       "sink + 3 recent frames; 40 heads x 128",
    3: "chunk_tiered: one streaming chunk at 1344x768 (3 latent frames x 1008 + 20 audio) over 256 prompt + "
       "sink + 12 frames pooled 4x4 + 9 frames pooled 2x2 + 3 full frames; 40 heads x 128",
    4: "clip: full 5 s clip, 30 latent frames x 1008 + 200 audio over themselves + 256 prompt; 40 heads x 128",
    5: "ragged: 20 sessions of the streaming chunk with segment lengths varied +-10%; 40 heads x 128",
}


def attention_bytes(win) -> int:
    """Algorithmic bytes of one attention launch: Q and O of the valid
    queries, K and V of the valid keys (bf16), each once."""
    q = int(win.q_len.sum().item())
    kv = int(win.lengths.sum())
    return 2 * win.H * win.D * (2 * q + 2 * kv)


def attention_flops(specs) -> float:
    from streaming_video_audio_b200.window import SessionPlan
    tot = 0.0
    for s in specs:
        p = SessionPlan(s)
        tot += 4.0 * p.chunk_len * sum(p.lengths.values()) * s.head_dim * s.n_heads
    return tot


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), \
            float(d["hbm_gbs"]), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.3)

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        rows = [r.split(",") for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def rank_sessions(config: int, rank: int):
    """(spec, seed) pairs a rank runs: every rank runs the whole workload on
    its own seeds (independent sessions; weak scaling, no data exchange)."""
    return [(s, seed + 1000 * rank) for s, seed in workloads.session_list(config)]


def aggregate(local_ms, flops_per_step: float, steps: int, world: int, group=None):
    """Max over ranks of each timing (ms), then whole-job throughput:
    TFLOP/s = world * flops_per_step * steps / max time.  `local_ms` is a
    list of this rank's [step-loop ms, end-to-end ms, attention ms]."""
    vals = torch.tensor([float(x) for x in local_ms], dtype=torch.float64)
    if group is not None or world > 1:
        import torch.distributed as dist
        if dist.get_backend(group) == "nccl":
            vals = vals.cuda()
        dist.all_reduce(vals, op=dist.ReduceOp.MAX, group=group)
    total_ms, e2e_ms, attn_ms = vals.cpu().tolist()
    return {"total_ms": total_ms, "e2e_ms": e2e_ms, "attn_ms": attn_ms,
            "value": world * flops_per_step * steps / (total_ms * 1e-3) / 1e12,
            "e2e_value": world * flops_per_step * steps / (e2e_ms * 1e-3) / 1e12}


def build_window(config: int, rank: int, device):
    from streaming_video_audio_b200.window import StreamingWindow
    sessions = rank_sessions(config, rank)
    specs = [s for s, _ in sessions]
    inputs = [workloads.draw_session(s, seed) for s, seed in sessions]
    win = StreamingWindow(specs, device=device)
    win.load_window(inputs)
    B, qc, H, D = win.B, win.q_cap, win.H, win.D
    chunk = []
    for name in ("q", "k", "v"):
        t = torch.zeros(B, qc, H, D, dtype=torch.bfloat16)
        for b, inp in enumerate(inputs):
            x = getattr(inp, name)
            t[b, :x.shape[0]] = x
        chunk.append(t)
    return specs, inputs, win, chunk


def attention_traffic(config: int):
    """DRAM bytes per attention launch from the committed ncu capture
    (profiles/attention_traffic.json), or None when the capture was taken on
    another workload or the kernel source has changed since."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "attention_traffic.json")
    if config != 3 or not os.path.exists(path):
        return None
    rec = json.load(open(path))
    src = os.path.join(ROOT, "streaming_video_audio_b200", "csrc")
    h = hashlib.sha256()
    for name in ("chunk_attention.cu", "sr_device.cuh"):
        h.update(open(os.path.join(src, name), "rb").read())
    if h.hexdigest()[:16] != rec.get("source_sha256_16"):
        return None
    return int(rec["dram_bytes_read"]) + int(rec["dram_bytes_write"])


def launches_in_steps(win, tiered: bool, steps: int) -> int:
    """Library kernel launches of `steps` steps from the window's current
    slide state: append, RoPE of q, RoPE of the window, attention (+ the
    split merge) per step, and the slide's pooling and append calls."""
    n = (4 + (1 if win.workspace is not None else 0)) * steps
    if tiered:
        ptr = dict(win.ring_ptr)
        for _ in range(steps):
            ops, ptr = win.slide_ops(ptr)
            n += len(ops)
    return n


def cpu_baseline(specs, inputs, target_s: float = 12.0):
    """The fp64 oracle as it stands, on the host cores: every head of a
    sample of chunk rows of the first session (window assembly, pooling and
    RoPE of every key included in each call).  A 64-row probe sizes the
    measured sample to about target_s seconds of CPU work."""
    import oracle
    from streaming_video_audio_b200.window import SessionPlan
    spec, inp = specs[0], inputs[0]
    rng = np.random.default_rng(0)
    order = rng.permutation(spec.chunk_len)

    def timed(n):
        rows = sorted(order[:n].tolist())
        t0 = time.perf_counter()
        oracle.session_reference(spec, inp, rows=rows)
        return rows, time.perf_counter() - t0

    # two probes separate the per-call cost (window assembly, pooling, RoPE of
    # every key) from the per-row cost, then one run of about target_s seconds
    _, t1 = timed(min(64, spec.chunk_len))
    rows, t2 = timed(min(128, spec.chunk_len))
    per_row = max((t2 - t1) / 64.0, 1e-4)
    fixed = max(t1 - 64 * per_row, 0.0)
    n = int(min(spec.chunk_len, max(128, (target_s - fixed) / per_row)))
    if n > len(rows):
        rows, dt = timed(n)
    else:
        dt = t2
    lkv = sum(SessionPlan(spec).lengths.values())
    fl = 4.0 * len(rows) * lkv * spec.head_dim * spec.n_heads
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{len(rows)} of {spec.chunk_len} chunk rows x all {spec.n_heads} heads of {spec.name} "
                      f"(window assembly, pooling and RoPE of every key included), {dt:.1f} s"}


def run_reference(args, rank, world):
    """Reference arm: the fp64 CPU oracle on the host cores, one bounded
    sample of the workload per step."""
    if rank != 0:
        return
    import oracle
    from streaming_video_audio_b200.window import SessionPlan
    sessions = workloads.session_list(args.config)
    spec, seed = sessions[0]
    inp = workloads.draw_session(spec, seed)
    lkv = sum(SessionPlan(spec).lengths.values())
    rows = list(range(0, spec.chunk_len, max(1, spec.chunk_len // 32)))[:32]

    def step(i):
        oracle.session_reference(spec, inp, heads=[i % spec.n_heads], rows=rows)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    fl = 4.0 * len(rows) * lkv * spec.head_dim * args.steps
    val = fl / dt / 1e12
    cores = oracle.num_threads()
    sample = f"per step: {len(rows)} chunk rows x 1 head of {spec.name} (full window assembly, pooling, RoPE)"
    line = {"metric": "chunk attention TFLOP/s (fp64 CPU oracle)", "value": val, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": CONFIG_DESC[args.config]},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=3, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="sr", choices=["sr", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    from streaming_video_audio_b200 import capi
    capi.load()   # fails loudly without the CUDA library
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    specs, inputs, win, chunk = build_window(args.config, rank, device)
    tiered = any(s.tiers for s in specs)
    q, k, v = (t.to(device) for t in chunk)
    stream = torch.cuda.current_stream()
    K, W = args.steps, args.warmup

    n_video = specs[0].chunk_video_tokens
    k_clean, v_clean = k[:, :n_video], v[:, :n_video]   # stand-in for the finished chunk's clean K/V

    def one_step(i, ev=None):
        if tiered:
            win.advance(k_clean, v_clean)
        win.append_chunk(k, v)
        win.rotate(q)
        if ev is not None:
            ev[0].record(stream)
        win.attend()
        if ev is not None:
            ev[1].record(stream)

    for i in range(W):
        one_step(i)
    torch.cuda.synchronize()
    win.check_status()

    launches = launches_in_steps(win, tiered, K)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(K):
        one_step(W + i, evs[i])
    stop.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    win.check_status()
    total_ms = start.elapsed_time(stop)
    attn_ms = [a.elapsed_time(b) for a, b in evs]

    # end to end through the public host-buffer API: every step uploads its
    # q, k, v from pinned host memory and downloads its o; HostStepPipeline
    # overlaps those transfers with the neighbouring steps' compute; the
    # slide takes the previous step's uploaded chunk as the clean frames
    from streaming_video_audio_b200.window import HostStepPipeline
    qh, kh, vh = (t.pin_memory() for t in chunk)
    ohs = [torch.empty(win.o.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    pipe = HostStepPipeline(win)
    for i in range(W):
        pipe.step(qh, kh, vh, ohs[i % 2], slide=tiered)
    pipe.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(K):
        pipe.step(qh, kh, vh, ohs[i % 2], slide=tiered)
    stream.wait_stream(pipe.copy)
    stream.wait_stream(pipe.copy_back)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    oh = ohs[0]
    if dist:
        dist.barrier()

    flops = attention_flops(specs)
    agg = aggregate([total_ms, e2e_ms, float(np.mean(attn_ms))], flops, K, world)
    total_ms, e2e_ms, attn_avg_ms = agg["total_ms"], agg["e2e_ms"], agg["attn_ms"]
    peak, peak_sus, hbm, peak_kind = peaks()
    if rank == 0:
        achieved = flops / (attn_avg_ms * 1e-3) / 1e12
        line = {
            "metric": "chunk attention TFLOP/s and ms per streaming step on 1 B200; fraction of BF16 peak",
            "value": agg["value"],
            "unit": "TFLOP/s",
            "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": total_ms / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": CONFIG_DESC[args.config], "config": args.config,
                       "sessions_per_gpu": len(specs), "q_tokens": [int(x) for x in win.q_len.tolist()][:4],
                       "kv_tokens": [int(x) for x in win.lengths.sum(axis=1)][:4],
                       "attention_tflop_per_step_per_gpu": flops / 1e12,
                       "l2": "inputs larger than L2: window K/V alone are "
                             f"{2 * win.k_att.numel() * 2 / 1e6:.0f} MB per GPU (L2 126 MB)",
                       "parallelism": f"replicas x{world}, sessions sharded by rank, no collective"},
            "roofline": {"bound": "tensor", "kernel": "chunk_attention_kernel<128>", "achieved": achieved,
                         "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "frac_of_sustained": achieved / peak_sus, "peak_kind": peak_kind,
                         "attention_ms": attn_avg_ms, "traffic": attention_traffic(args.config),
                         "algorithmic_bytes": attention_bytes(win)},
            "e2e": {"value": agg["e2e_value"], "unit": "TFLOP/s",
                    "ms_per_step": e2e_ms / K,
                    "h2d_bytes_per_step": sum(t.numel() * 2 for t in chunk),
                    "d2h_bytes_per_step": oh.numel() * 2},
            "clocks": clocks,
            "gpu_launches": launches,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(specs, inputs)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
