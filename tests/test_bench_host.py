"""Host-side logic of bench.py that decides what a JSON line reports: the clock
summary taken during the timed region, the algorithmic byte counts and the
workload overrides.  CPU only."""
import datetime

import bench
import synth


def _line(t, mhz, reasons=("Not Active",) * 4, max_mhz=1965):
    ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return f"{ts}, {mhz}, {max_mhz}, 900.5, 0x0000000000000000, " + ", ".join(reasons) + "\n"


def test_clock_summary_keeps_the_timed_window_only():
    t0 = 1_800_000_000.0
    lines = [_line(t0 - 1.0, 900.0),                      # before the region (warm-up): ignored
             _line(t0 + 0.1, 1960.0), _line(t0 + 0.2, 1950.0),
             _line(t0 + 0.3, 1800.0, ("Not Active", "Not Active", "Not Active", "Active")),
             "garbage line\n", "\n",
             _line(t0 + 5.0, 500.0, ("Active", "Not Active", "Not Active", "Not Active"))]  # after: ignored
    got = bench.summarize_clock_samples(lines, t0, t0 + 0.5)
    assert got["samples"] == 3
    assert got["sm_mhz"] == 1950.0 and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"]


def test_clock_summary_short_region_and_empty():
    t0 = 1_800_000_000.0
    # a region shorter than 0.3 s is widened by one sampling interval
    got = bench.summarize_clock_samples([_line(t0 + 0.15, 1900.0)], t0, t0 + 0.05)
    assert got["samples"] == 1 and got["sm_mhz"] == 1900.0
    got = bench.summarize_clock_samples([_line(t0 + 3.0, 1900.0)], t0, t0 + 0.05)
    assert got["samples"] == 0 and got["sm_mhz"] is None
    # the slowdown reasons that reject a run are reported by name
    bad = ("Active", "Active", "Active", "Not Active")
    got = bench.summarize_clock_samples([_line(t0 + 0.5, 1200.0, bad)], t0, t0 + 1.0)
    assert got["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_algorithmic_bytes():
    # scoring reads every key once (the fp32 score write is overhead, counted in the
    # measured traffic, not in the algorithmic bytes); K and V read and written per
    # kept key, plus its position read and written
    assert bench.score_bytes_per_key(2, 128) == 256 and bench.score_bytes_per_key(1, 128) == 128
    assert bench.kept_bytes(2, 128) == 1032 and bench.kept_bytes(1, 64) == 264
    assert bench.score_bytes_per_key(2, 256) == 512


def test_default_line_is_the_largest_single_gpu_workload():
    import sys
    argv = sys.argv
    try:
        sys.argv = ["bench.py"]
        a = bench.parse()
    finally:
        sys.argv = argv
    assert a.workload == "qwen3_32b_128k" and a.also == "qwen3_8b_32k"
    keys = {n: w.n_layers * w.batch * w.n_kv_heads * w.seq_len[1] for n, w in synth.WORKLOADS.items()
            if w.layout == "contig" and not n.startswith("sweep")}
    assert max(keys, key=keys.get) == a.workload


def test_also_summary_keeps_the_step_figures():
    line = {"value": 1.0, "unit": "keys/s", "ms_per_step": 0.5, "steps": 3, "config": {"workload": "x"},
            "roofline": {}, "path_roofline": {}, "clocks": {}, "gpu_launches": 12, "path": "split",
            "e2e": None, "diagnostics": {"a": 1}}
    got = bench.also_summary(line)
    assert "e2e" not in got and "diagnostics" not in got and got["value"] == 1.0


def test_workload_overrides_and_rank_shards():
    class A:
        head_dim, rope = 64, "interleaved"
    wl = bench.with_layout(synth.WORKLOADS["qwen3_8b_32k"], A)
    assert wl.head_dim == 64 and wl.interleaved and wl.n_layers == 36
    w0, w1 = bench.rank_workload(wl, 0, 2048), bench.rank_workload(wl, 1, 2048)
    assert w0.seed != w1.seed and w0.head_dim == w1.head_dim == 64
    cfg = bench.workload_config(wl, 2048, "post", "cuda_graph", "fp8")
    assert cfg["kv_elem"] == "fp8" and cfg["rope"] == "interleaved" and cfg["head_dim"] == 64
