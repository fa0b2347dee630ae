#!/usr/bin/env python
"""Throughput of TriAttention KV-cache compression on B200: keys scored + selected +
compacted per second, and the fraction of the HBM roofline.

One step = tri_score + tri_compact over the whole workload (every row of every
layer), inputs resident in HBM (larger than L2).  Calibration (tri_calib) is
offline and timed separately.  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload qwen3_32b_128k] [--also qwen3_8b_32k|none] [--budget B] [--key-mode post|pre]
                  [--elem bf16|fp8] [--head-dim 64|128|256] [--rope half|interleaved] [--no-variants]

The default line also carries the 32K workload's step ('also') and the same step
over a pre-RoPE cache and over an fp8 e4m3 cache ('variants'), step timings only.

N > 1 (under torchrun): every rank compacts its own cache of the same shape
(independent sequences; no collective on the data path), timing is the max
over ranks, value = keys of all ranks / that time (weak scaling).
--impl reference times the CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "keys scored+selected+compacted/sec per B200 and % of HBM roofline"
UNIT = "keys/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
ELEM_BYTES = {"bf16": 2, "fp8": 1}


def score_bytes_per_key(eb: int, d: int = 128) -> int:
    return d * eb  # read the key (the fp32 score write is overhead: it shows in the measured traffic)


def kept_bytes(eb: int, d: int = 128) -> int:
    return 4 * d * eb + 8  # read + write K and V of a kept key, read + write its position


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen3_32b_128k", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--also", default="qwen3_8b_32k", choices=sorted(synth.WORKLOADS) + ["none"],
                    help="a second workload timed in the same run (step timing only), reported under 'also'; "
                         "skipped with --layers, --budget or when it equals --workload")
    ap.add_argument("--budget", type=int, default=None)
    ap.add_argument("--layers", type=int, default=None,
                    help="first N layers only (small cases for profiling; not a bench line)")
    ap.add_argument("--key-mode", choices=["post", "pre"], default="post")
    ap.add_argument("--elem", choices=sorted(ELEM_BYTES), default="bf16",
                    help="K/V cache element type (fp8 = OCP e4m3, converted from the bf16 cache)")
    ap.add_argument("--head-dim", type=int, choices=[64, 128, 256], default=None,
                    help="override the workload's head dim (same heads and lengths)")
    ap.add_argument("--rope", choices=["half", "interleaved"], default=None,
                    help="override the workload's RoPE pairing")
    ap.add_argument("--launch", choices=["graph", "eager"], default="graph",
                    help="timed steps replay CUDA graphs of the calls (default) or call eagerly")
    ap.add_argument("--path", choices=["split", "fused"], default="split",
                    help="split: tri_score + tri_compact (the faster of the two on the 32K workload, by ~1%%); "
                         "fused: one tri_score_compact call per step (rows up to TRI_FUSED_MAX_ROW keys, scores "
                         "kept on chip, no score buffer)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the 32K workload's pre-RoPE and fp8 step timings reported under 'variants'")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    a = ap.parse_args()
    a.warmup = max(a.warmup, 3)
    return a


def workload_config(wl, B, key_mode, launch="eager", elem="bf16"):
    lo, hi = wl.seq_len
    eb = ELEM_BYTES[elem]
    return {"workload": wl.name, "layers": wl.n_layers, "q_heads": wl.n_q_heads,
            "kv_heads": wl.n_kv_heads, "head_dim": wl.head_dim, "rope_theta": wl.theta,
            "batch": wl.batch, "keys_per_head": lo if lo == hi else [lo, hi], "budget": B,
            "window": wl.window, "offsets": wl.n_offsets, "key_mode": key_mode + "_rope",
            "launch": launch,
            "layout": wl.layout, "kv_elem": elem, "rope": wl.rope_style,
            "l2": "inputs larger than L2: K+V %.1f GB read per step, no flush" % (
                2 * wl.head_dim * eb * wl.n_layers * wl.batch * wl.n_kv_heads * np.mean(wl.seq_len) / 1e9)}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            return float(json.load(fh)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def score_kernel_sha():
    h = hashlib.sha256()
    for f in ("score.cu", "score_common.cuh", "keys.cuh", "tri_internal.cuh"):
        with open(os.path.join(ROOT, "kv_cache_compression_calib_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(total_keys, elem="bf16"):
    """DRAM bytes per launch of the score kernel from the committed ncu summary, if it
    was taken on the current kernel source for this element type; else None."""
    path = os.path.join(ROOT, "profiles", "score_kernel_traffic.json")
    try:
        with open(path) as fh:
            rec = json.load(fh)
    except Exception:
        return None
    per = rec.get("by_elem", {}).get(elem)
    if rec.get("kernel_sha") != score_kernel_sha() or per is None:
        return None
    return float(per["dram_bytes_per_key"]) * total_keys


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms from before the
    warm-up until after the timed region; only samples stamped inside the timed
    region (widened by one interval when it is shorter than that) are reported."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.ident = str(device_index)

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.ident, "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t_begin, t_end):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        with open(self.path) as fh:
            lines = fh.readlines()
        os.unlink(self.path)
        return summarize_clock_samples(lines, t_begin, t_end)


def summarize_clock_samples(lines, t_begin, t_end):
    """Median SM clock, maximum clock and active throttle reasons of the nvidia-smi
    samples (lines of ClockSampler.FIELDS, csv without units) stamped inside
    [t_begin, t_end] (widened by 0.12 s when the region is shorter than 0.3 s);
    malformed lines are skipped."""
    rows = []
    for line in lines:
        p = [x.strip() for x in line.split(",")]
        if len(p) < 9:
            continue
        try:
            ts = datetime.datetime.strptime(p[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            rows.append((ts, float(p[1]), float(p[2]), p[5:9]))
        except ValueError:
            continue
    pad = 0.0 if t_end - t_begin >= 0.3 else 0.12
    win = [r for r in rows if t_begin - pad <= r[0] <= t_end + pad]
    if not win:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                "note": "timed region shorter than the sampling interval"}
    reasons = sorted({ClockSampler.REASONS[i] for r in win for i in range(4) if r[3][i].lower() == "active"})
    return {"sm_mhz": statistics.median(r[1] for r in win), "sm_max_mhz": max(r[2] for r in win),
            "reasons": reasons, "samples": len(win)}


# ------------------------------------------------------- multi-rank logic

def with_layout(wl, a):
    """The workload with --head-dim / --rope applied (same heads, lengths and budget)."""
    if a.head_dim:
        wl = wl.with_(head_dim=a.head_dim)
    if a.rope:
        wl = wl.with_(rope_style=a.rope)
    return wl


def rank_workload(wl, rank: int, B: int):
    """Rank r compacts its own independent cache of the same shape (other sequences):
    same workload, seed offset by the rank.  No rank reads another's rows."""
    return wl.with_(budget=B, seed=wl.seed + 7919 * rank)


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's time (all-reduce MAX; NCCL on GPUs, gloo on CPU)."""
    if world <= 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def throughput(keys_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job keys per second: every rank's keys over the slowest rank's step time."""
    return keys_per_rank * world / (ms_per_step / 1e3)


# ----------------------------------------------------------------- ours

def run_ours(a, rank, world, local_rank, workload=None, light=False):
    """One workload's bench line.  light: the step timing only (no end-to-end leg,
    CPU baseline or off-step diagnostics), for the extra workload of a run."""
    import kv_cache_compression_calib_b200 as tri

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl0 = synth.WORKLOADS[workload or a.workload]
    B = (a.budget if not light else None) or wl0.budget
    if a.layers:
        wl0 = wl0.with_(n_layers=min(a.layers, wl0.n_layers))
    wl0 = with_layout(wl0, a)
    wl = rank_workload(wl0, rank, B)
    key_mode = tri.TRI_KEYS_PRE_ROPE if a.key_mode == "pre" else tri.TRI_KEYS_POST_ROPE
    if wl.layout != "contig":
        return run_paged(a, tri, wl, B, rank, world, dev)
    cache = synth.make_contig(wl, dev, rotate=(a.key_mode == "post"))
    eb = ELEM_BYTES[a.elem]
    if a.elem == "fp8":
        cache.K = synth.to_fp8(cache.K)
        cache.V = synth.to_fp8(cache.V)
        torch.cuda.empty_cache()
    L, S, Hh = wl.n_layers, len(cache.lens), wl.n_kv_heads
    R, total = cache.n_rows, cache.total
    m = tri.model(L, wl.n_q_heads, Hh, wl.theta, head_dim=wl.head_dim,
                  rope_style=tri.TRI_ROPE_INTERLEAVED if wl.interleaved else tri.TRI_ROPE_HALF)
    D = wl.head_dim
    kv = tri.kv_contig(S, cache.row_off, total, tri.elem_type_of(cache.K))
    stream = torch.cuda.current_stream(dev)

    # offline calibration (timed separately, not part of a step)
    centres = torch.empty(L, wl.n_q_heads, D // 2, 2, dtype=torch.float32, device=dev)
    mnorm = torch.empty(L, wl.n_q_heads, D // 2, dtype=torch.float32, device=dev)
    tri.tri_calib(m, cache.qcal, wl.n_calib, centres, mnorm)
    torch.cuda.synchronize()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record()
    tri.tri_calib(m, cache.qcal, wl.n_calib, centres, mnorm)
    c1.record()
    torch.cuda.synchronize()
    calib_ms = c0.elapsed_time(c1)

    ws = tri.alloc_workspace(m, S, B, device=dev)
    scores = torch.empty(total, dtype=torch.float32, device=dev)
    Ko = torch.empty(R, B, D, dtype=cache.K.dtype, device=dev)
    Vo = torch.empty_like(Ko)
    po = torch.empty(R, B, dtype=torch.int32, device=dev)
    kept = torch.empty(R, B, dtype=torch.int32, device=dev)
    offsets = wl.offsets

    out_desc = tri.out_contig()
    max_row = int(np.diff(cache.row_off_np).max())
    fused = a.path == "fused"

    if fused:
        def score_call():  # the whole step: prep, fused score/select, gather
            tri.tri_score_compact(m, kv, cache.K, cache.V, cache.pos, centres, mnorm, cache.p_now, offsets, key_mode,
                                  B, wl.window, max_row, out_desc, Ko, Vo, po, kept, None, None, ws,
                                  torch.cuda.current_stream(dev))

        def compact_call():
            pass
    else:
        def score_call():  # on the current stream (the capture stream while capturing)
            tri.tri_score(m, kv, cache.K, cache.pos, centres, mnorm, cache.p_now, offsets, key_mode, scores, ws,
                          torch.cuda.current_stream(dev))

        def compact_call():
            tri.tri_compact(m, kv, scores, B, wl.window, cache.K, cache.V, cache.pos, out_desc, Ko, Vo, po, kept,
                            None, ws, torch.cuda.current_stream(dev))

    sampler = ClockSampler(local_rank)
    sampler.start()
    for _ in range(a.warmup):
        score_call()
        compact_call()
    torch.cuda.synchronize()
    st, flags = tri.tri_status_check(ws, stream)
    if st != 0:
        raise RuntimeError(f"device flags {flags:#x} after warm-up")
    if a.launch == "graph":
        g_score, g_compact = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_score):
            score_call()
        with torch.cuda.graph(g_compact):
            compact_call()
        do_score, do_compact = g_score.replay, g_compact.replay
        for _ in range(a.warmup):
            do_score()
            do_compact()
        torch.cuda.synchronize()
    else:
        do_score, do_compact = score_call, compact_call

    # ---- device-resident timed region
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    t0.record(stream)
    for i in range(a.steps):
        ev[i][0].record(stream)
        do_score()
        ev[i][1].record(stream)
        do_compact()
    t1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop(wall0, wall1)
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    score_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    st, flags = tri.tri_status_check(ws, stream)
    if st != 0:
        raise RuntimeError(f"device flags {flags:#x} in the timed region")

    lens_rows = np.diff(cache.row_off_np)
    keys_step = int(total)
    alg_bytes = float(np.sum(float(D) * eb * lens_rows + np.minimum(lens_rows, B) * kept_bytes(eb, D)))
    if key_mode == tri.TRI_KEYS_PRE_ROPE:
        alg_bytes += 4.0 * total
    ms_step = ms / a.steps
    value = throughput(keys_step, world, ms_step)

    diagnostics = {}
    if not light:
        diagnostics = time_diagnostics(tri, m, kv, cache, key_mode, wl, eb, dev, stream)
        diagnostics.update(time_attention(tri, m, cache, Ko, Vo, wl, B, eb, dev, stream))

    # ---- end to end through the public API: pinned host inputs, copies in the region
    e2e = None
    if not a.no_e2e and not light:
        e2e = run_e2e(a, tri, cache, centres, mnorm, key_mode, B, wl, stream, world, dev)

    # prep + score + select (the selection kernel copies the records itself when rows
    # average more than one 32768-slot chunk, else a gather kernel follows); fused:
    # prep + fused score/select + gather
    launches_per_step = 3 if fused or total > cache.n_rows * 32768 else 4
    peak, peak_kind = measured_peak()
    if fused:  # one call per step: its roofline is the whole path's
        score_bytes = alg_bytes
        kernel = "tri_score_compact (prep + fused score/select + gather kernels)"
        traffic = None
    else:
        score_bytes = score_bytes_per_key(eb, D) * total
        kernel = "tri_score (prep + score kernels)"
        traffic = (recorded_traffic(total, a.elem) if (D, wl.rope_style, a.key_mode) == (128, "half", "post")
                   else None)
    achieved = score_bytes / (score_ms / 1e3) / 1e9
    path_gbs = alg_bytes / (ms_step / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(wl, B, a.key_mode, "cuda_graph" if a.launch == "graph" else "eager", a.elem),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "kernel": kernel, "peak_kind": peak_kind,
                     "bytes_per_launch": score_bytes, "ms_per_launch": score_ms},
        "path_roofline": {"bytes_per_step": alg_bytes, "achieved_gbs": path_gbs,
                          "frac_of_measured": path_gbs / peak, "frac_of_8tbs": path_gbs / NOMINAL_HBM_GBS},
        "calib_ms": calib_ms,
        "diagnostics": diagnostics,
        "gpu_launches": launches_per_step * a.steps,
        "path": "fused" if fused else "split",
        "clocks": clocks,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not a.no_cpu_baseline and not light:
        line["cpu_baseline"] = cpu_baseline(wl, B, cache, a.cpu_seconds)
    return line


def also_summary(line):
    """The step figures of an extra workload's line (same clock, same run)."""
    keep = ("value", "unit", "ms_per_step", "steps", "config", "roofline", "path_roofline", "clocks",
            "gpu_launches", "path")
    return {k: line[k] for k in keep if k in line}


def run_paged(a, tri, wl, B, rank, world, dev):
    """The paged serving workload: a step is round 0 (every sequence's prefill,
    8K..32K keys per head in 16-token blocks, scored and compacted to B into a
    fresh block table) plus `wl.rounds` re-score rounds (the retained B keys and
    `wl.rescore_every` new decode tokens per head, scored and compacted into a
    fresh table).  The rounds are replayed on one steady-state input of the
    same shape as every later round (appending the decode tokens is the model's
    own KV write and stays outside the timed region)."""
    stream = torch.cuda.current_stream(dev)
    fused = a.path == "fused"
    S, Hh, bs, W, D = wl.batch, wl.n_kv_heads, wl.block_size, wl.window, wl.head_dim
    lens = wl.seq_lengths()
    pg = synth.make_paged(wl, dev, lens=lens)
    eb = 2
    if a.elem == "fp8":
        pg.K, pg.V = synth.to_fp8(pg.K), synth.to_fp8(pg.V)
        eb = 1
    et = tri.elem_type_of(pg.K)
    m = tri.model(1, wl.n_q_heads, Hh, wl.theta, head_dim=D,
                  rope_style=tri.TRI_ROPE_INTERLEAVED if wl.interleaved else tri.TRI_ROPE_HALF)
    qcal = synth.calib_queries(wl, 0, dev)[None].contiguous()
    c = torch.empty(1, wl.n_q_heads, D // 2, 2, device=dev)
    n = torch.empty(1, wl.n_q_heads, D // 2, device=dev)
    tri.tri_calib(m, qcal, wl.n_calib, c, n)
    new = wl.rescore_every
    ob = (B + new + bs - 1) // bs
    n_out = S * ob
    rng = np.random.default_rng(5)
    tables = [torch.as_tensor(rng.permutation(n_out).reshape(S, ob).astype(np.int32), device=dev) for _ in range(2)]
    outs = [(torch.zeros(1, n_out, bs, Hh, D, dtype=pg.K.dtype, device=dev),
             torch.zeros(1, n_out, bs, Hh, D, dtype=pg.K.dtype, device=dev),
             torch.full((1, n_out, bs, Hh), -1, dtype=torch.int32, device=dev)) for _ in range(2)]
    ws = tri.alloc_workspace(m, S, B, device=dev)
    kept = torch.empty(S * Hh, B, dtype=torch.int32, device=dev)

    def round_call(cur, p_now, K, V, P, table, nb, o):
        row_off = torch.as_tensor(synth.paged_row_offsets(cur, Hh), device=dev)
        total = int(synth.paged_row_offsets(cur, Hh)[-1])
        kv = tri.kv_paged(S, row_off, total, table, bs, nb, et)
        pn = torch.as_tensor(np.asarray(p_now), device=dev)
        scores = torch.empty(total, device=dev)
        Ko, Vo, Po = outs[o]
        max_row = int(np.max(cur))
        if fused:
            def call(st):
                # with a score buffer the library fuses the short rounds and runs round 0's
                # long prefills through the two-call path
                tri.tri_score_compact(m, kv, K, V, P, c, n, pn, wl.offsets, tri.TRI_KEYS_POST_ROPE, B, W, max_row,
                                      tri.out_paged(tables[o], bs, n_out), Ko, Vo, Po, kept, None, scores, ws, st)
        else:
            def call(st):
                tri.tri_score(m, kv, K, P, c, n, pn, wl.offsets, tri.TRI_KEYS_POST_ROPE, scores, ws, st)
                tri.tri_compact(m, kv, scores, B, W, K, V, P, tri.out_paged(tables[o], bs, n_out), Ko, Vo, Po,
                                kept, None, ws, st)
        return call, total, (kv, pn, scores, row_off)

    # round 0 on the prefill; then a steady-state input: its output plus `new` decode tokens
    call0, keys0, keep0 = round_call(lens, lens, pg.K, pg.V, pg.pos, pg.block_table.to(dev), pg.K.shape[0], 0)
    call0(stream)
    torch.cuda.synchronize()
    cur = np.minimum(lens, B)
    Kn, Vn = synth.decode_keys(wl, 0, 0, lens, new, dev)
    if a.elem == "fp8":
        Kn, Vn = synth.to_fp8(Kn), synth.to_fp8(Vn)
    tbl0 = tables[0].cpu().numpy()
    K1, V1, P1 = outs[0]
    for s_ in range(S):
        j = np.arange(int(cur[s_]), int(cur[s_]) + new)
        blk = torch.as_tensor(tbl0[s_, j // bs].astype(np.int64), device=dev)
        slot = torch.as_tensor(j % bs, device=dev)
        K1[0, blk, slot] = Kn[s_]
        V1[0, blk, slot] = Vn[s_]
        P1[0, blk, slot] = torch.arange(int(lens[s_]), int(lens[s_]) + new, device=dev, dtype=torch.int32)[:, None]
    cur1 = cur + new
    call1, keys1, keep1 = round_call(cur1, lens + new, K1, V1, P1, tables[0], n_out, 1)

    graphs = []
    for call in (call0, call1):
        for _ in range(a.warmup):
            call(stream)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call(torch.cuda.current_stream())
        graphs.append(g)
    st, flags = tri.tri_status_check(ws, stream)
    if st != 0:
        raise RuntimeError(f"device flags {flags:#x} after warm-up")
    for _ in range(a.warmup):
        graphs[0].replay()
        for _ in range(wl.rounds):
            graphs[1].replay()
    sampler = ClockSampler(dev.index or 0)
    sampler.start()
    ev0 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    t0.record(stream)
    for i in range(a.steps):
        ev0[i][0].record(stream)
        graphs[0].replay()
        ev0[i][1].record(stream)
        for _ in range(wl.rounds):
            graphs[1].replay()
    t1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop(wall0, wall1)
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    r0_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev0)
    st, flags = tri.tri_status_check(ws, stream)
    if st != 0:
        raise RuntimeError(f"device flags {flags:#x} in the timed region")
    ms_step = ms / a.steps
    keys_step = keys0 + wl.rounds * keys1
    rows0 = np.repeat(lens, Hh)
    rows1 = np.repeat(cur1, Hh)
    kb = kept_bytes(eb, D)
    bytes0 = float(np.sum(float(D) * eb * rows0 + np.minimum(rows0, B) * kb))
    bytes1 = float(np.sum(float(D) * eb * rows1 + np.minimum(rows1, B) * kb))
    alg_bytes = bytes0 + wl.rounds * bytes1
    r1_ms = (ms_step - r0_ms) / wl.rounds
    peak, peak_kind = measured_peak()
    line = {
        "metric": METRIC, "value": throughput(keys_step, world, ms_step), "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": dict(workload_config(wl, B, "post", "cuda_graph", a.elem), rounds=wl.rounds, new_tokens=new,
                       keys_round0=int(keys0), keys_per_round=int(keys1)),
        "roofline": {"bound": "hbm", "achieved": bytes0 / (r0_ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": bytes0 / (r0_ms / 1e3) / 1e9 / peak, "traffic": None,
                     "kernel": "round 0 (prep + fused score/select + gather kernels)" if fused else
                     "round 0 (prep + score + select + gather kernels)", "peak_kind": peak_kind,
                     "bytes_per_launch": bytes0, "ms_per_launch": r0_ms},
        "path_roofline": {"bytes_per_step": alg_bytes, "achieved_gbs": alg_bytes / (ms_step / 1e3) / 1e9,
                          "frac_of_measured": alg_bytes / (ms_step / 1e3) / 1e9 / peak,
                          "frac_of_8tbs": alg_bytes / (ms_step / 1e3) / 1e9 / NOMINAL_HBM_GBS,
                          "round0_ms": r0_ms, "round_ms": r1_ms,
                          "round_frac_of_measured": bytes1 / (r1_ms / 1e3) / 1e9 / peak},
        "gpu_launches": 3 * (1 + wl.rounds) * a.steps,
        "clocks": clocks,
        "e2e": None,
        "path": "fused" if fused else "split",
    }
    return line


def graph_time(call, stream, reps):
    """Mean device time of one `call(stream)` (its kernels captured once in a CUDA
    graph and replayed `reps` times between CUDA events), so the host's launch
    rate does not set the pace of short calls."""
    call(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(torch.cuda.current_stream())
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def time_diagnostics(tri, m, kv, cache, key_mode, wl, eb, dev, stream, reps=5):
    """Off-step calls, timed by CUDA graph replay (mean of `reps` after one warm-up):
    the key-centre pass over the whole cache (reads every key once: d x elem bytes
    per key) and one online centre update with 64 new queries per head."""
    D, L, Hq = wl.head_dim, wl.n_layers, wl.n_q_heads
    R, S = cache.n_rows, len(cache.lens)
    kc = torch.empty(R, D // 2, 2, device=dev)
    kn = torch.empty(R, D // 2, device=dev)
    kws = tri.alloc_key_centres_workspace(m, S, device=dev)
    q = cache.qcal[:, :, :64].contiguous()
    sums = torch.zeros(L, Hq, D // 2, 3, dtype=torch.float64, device=dev)
    weight = torch.zeros(L, Hq, dtype=torch.float64, device=dev)
    uc = torch.empty(L, Hq, D // 2, 2, device=dev)
    un = torch.empty(L, Hq, D // 2, device=dev)

    kc_ms = graph_time(lambda s: tri.tri_key_centres(m, kv, cache.K, cache.pos, key_mode, kc, kn, kws, s), stream,
                       reps)
    st, flags = tri.tri_status_check(kws, stream)
    if st != 0:
        raise RuntimeError(f"device flags {flags:#x} in the key-centre pass")
    up_ms = graph_time(lambda s: tri.tri_calib_update(m, q, 64, 0.99, sums, weight, uc, un, s), stream, reps)
    peak, kind = measured_peak()
    kc_bytes = float(cache.total) * D * eb
    return {"key_centres_ms": kc_ms, "key_centres_bytes": kc_bytes,
            "key_centres_gbs": kc_bytes / (kc_ms / 1e3) / 1e9,
            "key_centres_frac": kc_bytes / (kc_ms / 1e3) / 1e9 / peak, "peak_kind": kind,
            "calib_update_ms": up_ms, "calib_update_queries_per_head": 64}


def time_attention(tri, m, cache, Ko, Vo, wl, B, eb, dev, stream, reps=10):
    """Decode attention (one query per query head) over the compacted [R][B] cache
    the step wrote, timed by CUDA graph replay; algorithmic bytes = K and V of every
    kept key + queries + fp32 outputs.  Reported only when every row filled its
    budget (the compacted rows are then end to end)."""
    lens_rows = np.diff(cache.row_off_np)
    if lens_rows.min() < B:
        return {}
    import math
    D, L, Hq, S = wl.head_dim, wl.n_layers, wl.n_q_heads, len(cache.lens)
    R = cache.n_rows
    kvc = tri.kv_contig(S, torch.arange(R + 1, device=dev, dtype=torch.int64) * B, R * B, tri.elem_type_of(Ko))
    q = synth.decode_queries(wl, 0, np.asarray(cache.lens), dev)[None].expand(L, -1, -1, -1).contiguous()
    out = torch.empty(L, S, Hq, D, device=dev)
    lse = torch.empty(L, S, Hq, device=dev)
    ws = tri.alloc_attention_workspace(m, S, device=dev)
    scale = 1.0 / math.sqrt(D)
    ms = graph_time(lambda s: tri.tri_decode_attention(m, kvc, Ko, Vo, q, scale, out, lse, ws, s), stream, reps)
    st, flags = tri.tri_status_check(ws, stream)
    if st != 0:
        raise RuntimeError(f"device flags {flags:#x} in decode attention")
    nbytes = float(R) * B * 2 * D * eb + q.numel() * 2 + out.numel() * 4 + lse.numel() * 4
    peak, _ = measured_peak()
    res = {"decode_attention_ms": ms, "decode_attention_bytes": nbytes,
           "decode_attention_gbs": nbytes / (ms / 1e3) / 1e9,
           "decode_attention_frac": nbytes / (ms / 1e3) / 1e9 / peak,
           "decode_attention_l2": "the compacted K+V (%.0f MB) fit in L2: timed warm" % (R * B * 2 * D * eb / 1e6)
           if R * B * 2 * D * eb < 100e6 else "compacted K+V larger than L2"}
    if eb == 2 and D == 128 and wl.group <= 16:
        # the tensor-memory kernel on the same cache and queries, timed beside it
        ms_tc = graph_time(lambda s: tri.tri_decode_attention_tc(m, kvc, Ko, Vo, q, scale, out, lse, ws, s),
                           stream, reps)
        st, flags = tri.tri_status_check(ws, stream)
        if st != 0:
            raise RuntimeError(f"device flags {flags:#x} in tensor-memory decode attention")
        res.update({"decode_attention_tc_ms": ms_tc,
                    "decode_attention_tc_frac": nbytes / (ms_tc / 1e3) / 1e9 / peak})
    return res


HOST_CACHE_BYTES = 24 << 30  # pinned host memory the end-to-end leg may hold for the cache


def run_e2e(a, tri, cache, centres, mnorm, key_mode, B, wl, stream, world, dev):
    """End to end through the public calls with the cache on the host, streamed
    layer by layer.  Every step, for every layer: K and the positions are copied
    from pinned host memory into the layer's device region on a copy stream
    (overlapping the previous layer's calls), then tri_score and tri_compact run
    on the layer; the gather reads only the kept records of V from pinned host
    memory and writes the compacted K, V and positions straight into pinned host
    buffers; p_now is copied in at the start and the kept indices read back at
    the end.  The calibration (offline, like the model's weights) stays on the
    device.  The pinned host cache holds at most HOST_CACHE_BYTES of layers (the
    host has far less RAM than a 128K cache): layer l streams from host layer
    l mod h, so every byte of every layer still crosses the link each step."""
    L, S, Hh, D = wl.n_layers, len(cache.lens), wl.n_kv_heads, wl.head_dim
    rpl = S * Hh
    ro = cache.row_off_np
    eb = cache.K.element_size()
    et = tri.elem_type_of(cache.K)
    m1 = tri.model(1, wl.n_q_heads, Hh, wl.theta, head_dim=D,
                   rope_style=tri.TRI_ROPE_INTERLEAVED if wl.interleaved else tri.TRI_ROPE_HALF)
    spans = [(int(ro[l * rpl]), int(ro[(l + 1) * rpl])) for l in range(L)]
    kvs = []
    for l, (a0, a1) in enumerate(spans):
        roff = torch.as_tensor(ro[l * rpl:(l + 1) * rpl + 1] - a0, device=dev)
        kvs.append(tri.kv_contig(S, roff, a1 - a0, et))
    layer_bytes = max(a1 - a0 for a0, a1 in spans) * (2 * D * eb + 4)
    hl = int(max(1, min(L, HOST_CACHE_BYTES // max(layer_bytes, 1))))
    try:
        hK, hV, hP = [], [], []
        for a0, a1 in spans[:hl]:
            for lst, src in ((hK, cache.K), (hV, cache.V), (hP, cache.pos)):
                h = torch.empty(src[a0:a1].shape, dtype=src.dtype, pin_memory=True)
                h.copy_(src[a0:a1])
                lst.append(h)
        oK = [torch.empty(rpl, B, D, dtype=cache.K.dtype, pin_memory=True) for _ in range(L)]
        oV = [torch.empty(rpl, B, D, dtype=cache.K.dtype, pin_memory=True) for _ in range(L)]
        oP = [torch.empty(rpl, B, dtype=torch.int32, pin_memory=True) for _ in range(L)]
        hpn = cache.p_now.cpu().pin_memory()
        kept = torch.empty(L * rpl, B, dtype=torch.int32, device=dev)
        okept = torch.empty(kept.shape, dtype=kept.dtype, pin_memory=True)
    except RuntimeError as e:
        return {"value": None, "unit": UNIT, "skipped": f"pinned host buffers: {e}"[:200]}
    scores = torch.empty(cache.total, dtype=torch.float32, device=dev)
    ws = tri.alloc_workspace(m1, S, B, device=dev)
    copy = torch.cuda.Stream(dev)
    ready = [torch.cuda.Event() for _ in range(L)]
    done = [torch.cuda.Event() for _ in range(L)]
    out_desc = tri.out_contig()

    def step():
        cache.p_now.copy_(hpn, non_blocking=True)
        for l, (a0, a1) in enumerate(spans):
            h = l % hl
            with torch.cuda.stream(copy):
                copy.wait_event(done[l])  # the previous step's calls on this layer are done
                cache.K[a0:a1].copy_(hK[h], non_blocking=True)
                cache.pos[a0:a1].copy_(hP[h], non_blocking=True)
                ready[l].record(copy)
            stream.wait_event(ready[l])
            Kl, Pl = cache.K[a0:a1], cache.pos[a0:a1]
            tri.tri_score(m1, kvs[l], Kl, Pl, centres[l:l + 1], mnorm[l:l + 1], cache.p_now, wl.offsets, key_mode,
                          scores[a0:a1], ws, stream)
            tri.tri_compact(m1, kvs[l], scores[a0:a1], B, wl.window, Kl, hV[h], Pl, out_desc, oK[l], oV[l], oP[l],
                            kept[l * rpl:(l + 1) * rpl], None, ws, stream)
            done[l].record(stream)
        okept.copy_(kept, non_blocking=True)

    lens = np.diff(np.asarray(ro, dtype=np.int64))
    n_kept = int(np.minimum(lens, B).sum())
    rb = D * eb
    h2d = sum((a1 - a0) * (rb + 4) for a0, a1 in spans) + hpn.numel() * 8 + n_kept * rb
    d2h = okept.numel() * 4 + n_kept * (2 * rb + 4)
    est_s = h2d / 40e9
    steps = max(2, min(a.steps, 10, int(8.0 / max(est_s, 1e-3))))
    step()
    torch.cuda.synchronize()
    st, flags = tri.tri_status_check(ws, stream)
    if st != 0:
        raise RuntimeError(f"device flags {flags:#x} in the end-to-end leg")
    if world > 1:
        torch.distributed.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    copy.wait_event(t0)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    return {"value": throughput(cache.total, world, ms / steps), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": ms / steps, "copies_declared": True,
            "host_cache": f"{hl} of {L} layers of K, V and positions in pinned host memory; layer l streams from "
                          f"host layer l mod {hl}",
            "host_records": "V read and the compacted cache written in pinned host memory by the gather",
            "calls_per_step": f"tri_score + tri_compact per layer ({L} layers)"}


# ------------------------------------------------------- CPU oracle leg

def oracle_sample(wl, B, K_rows, V_rows, pos_rows, cs, ms, rows_meta, seconds, max_rows):
    """Time the oracle (collapsed score + select + gather) on rows until `seconds` pass.

    K_rows/V_rows hold the stored bits (int16 for bf16, uint8 for fp8)."""
    import oracle

    keys = 0
    n_rows = 0
    t0 = time.perf_counter()
    for i in range(max_rows):
        j = i % len(rows_meta)
        h, p_now = rows_meta[j]
        Kb = K_rows[j]
        Kf = oracle.e4m3_bits_to_f64(Kb) if Kb.dtype == np.uint8 else oracle.bf16_bits_to_f64(Kb)
        s = oracle.row_scores(wl.theta, cs, ms, h, wl.group, Kf, pos_rows[j], True, p_now, wl.offsets,
                              "collapsed", wl.interleaved)
        kept = oracle.select(s, B, wl.window)
        oracle.gather(K_rows[j], kept)
        oracle.gather(V_rows[j], kept)
        oracle.gather(pos_rows[j], kept)
        keys += len(s)
        n_rows += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return keys, n_rows, dt


def cpu_baseline(wl, B, cache, seconds):
    import oracle
    from tests import harness as H

    Hh = wl.n_kv_heads
    rows = list(range(min(Hh, cache.n_rows)))  # layer 0, sequence 0, every KV head
    K_rows, V_rows, pos_rows, meta = [], [], [], []
    for r in rows:
        a, b = cache.row_off_np[r], cache.row_off_np[r + 1]
        K_rows.append(H.raw_bits(cache.K[a:b]))
        V_rows.append(H.raw_bits(cache.V[a:b]))
        pos_rows.append(cache.pos[a:b].cpu().numpy().astype(np.int64))
        _, s, h = cache.row_lhs(r)
        meta.append((h, int(cache.lens[s])))
    cs, ms = H.oracle_calibration(cache.qcal[:1], wl.interleaved)
    keys, n_rows, dt = oracle_sample(wl, B, K_rows, V_rows, pos_rows, cs[0], ms[0], meta, seconds, 64)
    return {"value": keys / dt, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n_rows} rows x {len(K_rows[0])} keys of layer 0 (score collapsed fp64 + select + gather), "
                      f"{dt:.1f} s"}


def run_reference(a, rank, world):
    import oracle
    from tests import harness as H

    wl0 = synth.WORKLOADS[a.workload]
    B = a.budget or wl0.budget
    wl = with_layout(wl0.with_(budget=B), a)
    cache = synth.make_contig(wl, "cpu", layers=[0], lens=wl.seq_lengths()[:1])
    if a.elem == "fp8":
        cache.K = synth.to_fp8(cache.K)
        cache.V = synth.to_fp8(cache.V)
    Hh = wl.n_kv_heads
    K_rows, V_rows, pos_rows, meta = [], [], [], []
    for r in range(Hh):
        a_, b_ = cache.row_off_np[r], cache.row_off_np[r + 1]
        K_rows.append(H.raw_bits(cache.K[a_:b_]))
        V_rows.append(H.raw_bits(cache.V[a_:b_]))
        pos_rows.append(cache.pos[a_:b_].numpy().astype(np.int64))
        meta.append((r % Hh, int(cache.lens[0])))
    cs, ms = H.oracle_calibration(cache.qcal, wl.interleaved)
    for i in range(a.warmup):
        oracle_sample(wl, B, K_rows[i % Hh:i % Hh + 1], V_rows[i % Hh:i % Hh + 1], pos_rows[i % Hh:i % Hh + 1],
                      cs[0], ms[0], meta[i % Hh:i % Hh + 1], 0.0, 1)
    keys = 0
    t0 = time.perf_counter()
    for i in range(a.steps):
        j = i % Hh
        k, _, _ = oracle_sample(wl, B, K_rows[j:j + 1], V_rows[j:j + 1], pos_rows[j:j + 1], cs[0], ms[0],
                                meta[j:j + 1], 0.0, 1)
        keys += k
    dt = time.perf_counter() - t0
    value = keys / dt
    sample = f"1 row ({len(K_rows[0])} keys) of layer 0 per step (score collapsed fp64 + select + gather)"
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": dt / a.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": workload_config(wl, B, "post", "cuda_graph" if a.launch == "graph" else "eager", a.elem),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    a = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if a.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(a, rank, world)), flush=True)
        return
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(a, rank, world, local_rank)
        if a.also != "none" and a.also != a.workload and not a.layers and not a.budget:
            import gc

            gc.collect()
            torch.cuda.empty_cache()
            line["also"] = also_summary(run_ours(a, rank, world, local_rank, workload=a.also, light=True))
        if not a.no_variants and a.key_mode == "post" and a.elem == "bf16" and a.path == "split" \
                and not a.layers and not a.budget and a.head_dim is None and a.rope is None:
            # the same 32K step with a pre-RoPE cache and with an fp8 e4m3 cache
            import copy
            import gc

            variants = {}
            for name, field, val in (("pre_rope", "key_mode", "pre"), ("fp8", "elem", "fp8")):
                gc.collect()
                torch.cuda.empty_cache()
                b = copy.copy(a)
                setattr(b, field, val)
                variants[name] = also_summary(run_ours(b, rank, world, local_rank, workload="qwen3_8b_32k",
                                                       light=True))
            line["variants"] = variants
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
