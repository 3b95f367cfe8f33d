"""Host-side pieces of bench.py (CPU only): clock-sample summaries and the
launch count of the timed steps."""
import time

import bench


def _line(ts, sm, reasons=("Not Active",) * 4):
    stamp = time.strftime("%Y/%m/%d %H:%M:%S", time.localtime(ts)) + ".250"
    return ", ".join([stamp, "0", str(sm), "1965", "900.00", "0x0"] + list(reasons))


def test_clock_summary_keeps_the_timed_window():
    t = int(time.time()) + 0.25   # the stamps carry whole seconds + .250: keep t on that grid
    text = "\n".join([_line(t - 3, 600), _line(t - 1, 1800, ("Not Active", "Not Active", "Not Active", "Active")),
                      _line(t, 1700), _line(t + 5, 1965)])
    s = bench.ClockSampler.summarize(text, t - 1.5, t + 1)
    assert s["samples"] == 2 and s["in_timed_region"]
    assert s["sm_mhz"] == 1750.0 and s["sm_max_mhz"] == 1965.0 and s["reasons"] == ["sw_power_cap"]
    s = bench.ClockSampler.summarize(text, t + 10, t + 11)      # window without samples: all, flagged
    assert s["samples"] == 4 and not s["in_timed_region"]
    assert bench.ClockSampler.summarize("") is None
    assert bench.ClockSampler.summarize("garbage line\n") is None


def test_nvml_sample_summary_decodes_reason_bits():
    t = 1000.0
    samples = [(t - 1, 1000, 1965, 0x0), (t + 0.001, 1900, 1965, 0x4), (t + 0.003, 1800, 1965, 0x4 | 0x40),
               (t + 0.005, 1965, 1965, 0x1), (t + 2, 500, 1965, 0x8)]
    s = bench.ClockSampler.summarize_samples(samples, t, t + 0.01)
    assert s["samples"] == 3 and s["in_timed_region"] and s["sm_mhz"] == 1900.0
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]   # 0x1 (idle) is not a reason kept
    s = bench.ClockSampler.summarize_samples(samples, t + 10, t + 11)
    assert s["samples"] == 5 and not s["in_timed_region"] and "hw_slowdown" in s["reasons"]
    assert bench.ClockSampler.summarize_samples([]) is None


def test_await_sample_is_bounded():
    import threading
    import time
    s = object.__new__(bench.ClockSampler)
    s.thread = None
    s.await_sample(5.0)                       # nvidia-smi fallback: nothing to wait for
    s.thread, s.fresh = object(), threading.Event()
    t = time.time()
    s.await_sample(0.02)                      # no sample comes: gives up after the timeout
    assert 0.015 <= time.time() - t < 1.0
    s.fresh.set()
    t = time.time()
    s.await_sample(5.0)                       # a sample inside the region: returns at once
    assert time.time() - t < 0.5


def test_launch_count_follows_the_slide_plan():
    import workloads
    from streaming_video_audio_b200.window import StreamingWindow
    spec = workloads.scaled(workloads.CHUNK_TIERED, n_heads=1, head_dim=128, prompt_len=8, chunk_audio_tokens=4)
    win = StreamingWindow([spec], device="cpu")
    win._ring_setup(3)
    # CPU window: no split workspace -> 4 launches per step (append, 2 RoPE, attention) + 4 for the slide
    # (clock advance, two pooling boundaries, the clean-frame append)
    assert bench.launches_in_steps(win, True, 10) == 10 * (4 + 4)
    assert bench.launches_in_steps(win, False, 10) == 40


class _Ev:
    def __init__(self, t):
        self.t = t

    def elapsed_time(self, other):
        return other.t - self.t


def test_call_breakdown_sums_split_calls_and_averages_steps():
    e = [_Ev(x) for x in (0.0, 0.01, 0.03, 0.05, 0.55)]
    step = [("pool a->b", 100, e[0], e[1]), ("pool a->b", 50, e[1], e[2]), ("rope", 300, e[2], e[3]),
            ("attention", None, e[3], e[4])]
    rows = {n: (ms, nb) for n, ms, nb in bench.call_breakdown([step, step])}
    assert abs(rows["pool a->b"][0] - 0.03) < 1e-12 and rows["pool a->b"][1] == 150
    assert abs(rows["attention"][0] - 0.5) < 1e-12
    blk = bench.hbm_block(bench.call_breakdown([step]), 6556.0, "measured")
    assert [r["call"] for r in blk["calls"]] == ["pool a->b", "rope"]          # attention is not HBM-bound
    assert abs(blk["calls"][1]["achieved"] - 300 / 0.02e-3 / 1e9) < 1e-9
    assert abs(blk["step_ms_sum_of_calls"] - 0.55) < 1e-12
