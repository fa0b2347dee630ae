"""fp8 (OCP e4m3) KV caches: scoring reads 128-byte keys, compaction moves
128-byte records.  Parity as for bf16: scores against the literal oracle on the
exactly decoded fp8 keys (1e-4 of the series bound), selection bit-exact on
identical fp32 scores, compaction bit-exact given the index set."""
import numpy as np
import pytest
import torch

import kv_cache_compression_calib_b200 as tri
import oracle
import synth
from tests import harness as H
from tests.test_gpu_parity import model_of, oracle_centres

pytestmark = pytest.mark.gpu
DEV = "cuda"
FP8 = tri.TRI_ELEM_FP8_E4M3


def fp8_cache(wl, lens=None, rotate=True, layers=None):
    host = synth.make_contig(wl, "cpu", lens=lens, rotate=rotate, layers=layers)
    host.K = synth.to_fp8(host.K)
    host.V = synth.to_fp8(host.V)
    return host


def oracle_scores_fp8(host, cs, ms, post_rope=True, tier="literal"):
    wl = host.wl
    K = H.to_f64(host.K)
    pos = host.pos.numpy().astype(np.int64)
    ref = np.full(host.total, np.nan)
    bound = np.full(host.total, np.nan)
    for r in range(host.n_rows):
        li, s, h = host.row_lhs(r)
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        if a == b:
            continue
        ref[a:b] = oracle.row_scores(wl.theta, cs[li], ms[li], h, wl.group, K[a:b], pos[a:b], post_rope,
                                     int(host.lens[s]), wl.offsets, tier)
        bound[a:b] = H.series_bound(wl.theta, cs[li], ms[li], h, wl.group, K[a:b], wl.offsets)
    return ref, bound


def run(host, cs, ms, B, W, key_mode=tri.TRI_KEYS_POST_ROPE, scores=None):
    wl = host.wl
    m = model_of(wl, len(host.layers))
    S = len(host.lens)
    R = host.n_rows
    ro = host.row_off.to(DEV)
    kv = tri.kv_contig(S, ro, host.total, FP8)
    K, V, pos, pn = host.K.to(DEV), host.V.to(DEV), host.pos.to(DEV), host.p_now.to(DEV)
    ws = tri.alloc_workspace(m, S, B)
    if scores is None:
        scores = torch.full((max(host.total, 1),), float("nan"), device=DEV)
        tri.tri_score(m, kv, K, pos, torch.tensor(cs, dtype=torch.float32, device=DEV),
                      torch.tensor(ms, dtype=torch.float32, device=DEV), pn, wl.offsets, key_mode, scores, ws)
    else:
        scores = torch.tensor(scores, dtype=torch.float32, device=DEV)
    Ko = torch.zeros(R, B, 128, dtype=torch.float8_e4m3fn, device=DEV)
    Vo = torch.zeros_like(Ko)
    po = torch.full((R, B), -1, dtype=torch.int32, device=DEV)
    kept = torch.full((R, B), -1, dtype=torch.int32, device=DEV)
    tri.tri_compact(m, kv, scores, B, W, K, V, pos, tri.out_contig(), Ko, Vo, po, kept, None, ws)
    st, flags = tri.tri_status_check(ws)
    assert st == 0, flags
    return scores.cpu().numpy().astype(np.float64), H.raw_bits(Ko), H.raw_bits(Vo), po.cpu().numpy(), \
        kept.cpu().numpy()


@pytest.mark.parametrize("rotate,mode", [(True, tri.TRI_KEYS_POST_ROPE), (False, tri.TRI_KEYS_PRE_ROPE)])
def test_fp8_scores_selection_gather(rotate, mode):
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="fp8", batch=3, n_calib=128)
    lens = [4096, 1000, 33]
    host = fp8_cache(wl, lens=lens, rotate=rotate)
    cs, ms = oracle_centres(host)
    ref, bound = oracle_scores_fp8(host, cs, ms, post_rope=(mode == tri.TRI_KEYS_POST_ROPE))
    B, W = 512, 64
    got, *_ = run(host, cs, ms, B, W, key_mode=mode)
    assert H.score_error(got[:host.total], ref, bound) <= 1e-4
    # exact selection and compaction on the oracle's fp32 scores
    ref32 = H.as_f32_exact(ref)
    _, Kob, Vob, pob, kept = run(host, cs, ms, B, W, key_mode=mode, scores=ref32)
    Kb, Vb, pb = H.raw_bits(host.K), H.raw_bits(host.V), host.pos.numpy()
    for r in range(host.n_rows):
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        sel = oracle.select(ref32[a:b], B, W)
        n = len(sel)
        np.testing.assert_array_equal(kept[r, :n], sel)
        np.testing.assert_array_equal(Kob[r, :n], oracle.gather(Kb[a:b], sel))
        np.testing.assert_array_equal(Vob[r, :n], oracle.gather(Vb[a:b], sel))
        np.testing.assert_array_equal(pob[r, :n], oracle.gather(pb[a:b], sel))


def test_fp8_paged():
    wl = synth.WORKLOADS["paged_16seq"].with_(name="fp8paged", batch=3, n_calib=64)
    lens = np.array([300, 2100, 1024])
    p = synth.make_paged(wl, "cpu", lens=lens)
    p.K = synth.to_fp8(p.K)
    p.V = synth.to_fp8(p.V)
    qcal = synth.calib_queries(wl, 0, "cpu")[None]
    cs, ms = H.oracle_calibration(qcal)
    cs, ms = H.as_f32_exact(cs), H.as_f32_exact(ms)
    S, Hh, bs = len(lens), wl.n_kv_heads, wl.block_size
    row_off = synth.paged_row_offsets(lens, Hh)
    total = int(row_off[-1])
    Kf = H.to_f64(p.K).reshape(-1, 128)
    Kb = H.raw_bits(p.K).reshape(-1, 128)
    posf = p.pos.numpy().reshape(-1)
    ref = np.empty(total)
    recs = []
    for s in range(S):
        j = np.arange(int(lens[s]))
        blk = p.block_table_np[s, j // bs].astype(np.int64)
        for h in range(Hh):
            rec = (blk * bs + j % bs) * Hh + h
            recs.append(rec)
            r = s * Hh + h
            ref[row_off[r]:row_off[r + 1]] = oracle.row_scores(wl.theta, cs[0], ms[0], h, wl.group, Kf[rec],
                                                               posf[rec].astype(np.int64), True, int(lens[s]),
                                                               wl.offsets, "collapsed")
    m = model_of(wl, 1)
    kv = tri.kv_paged(S, torch.as_tensor(row_off, device=DEV), total, p.block_table.to(DEV), bs, p.K.shape[0],
                      FP8)
    ws = tri.alloc_workspace(m, S, 256)
    scores = torch.empty(total, device=DEV)
    Kd, Vd, pd = p.K.to(DEV), p.V.to(DEV), p.pos.to(DEV)
    tri.tri_score(m, kv, Kd, pd, torch.tensor(cs, dtype=torch.float32, device=DEV),
                  torch.tensor(ms, dtype=torch.float32, device=DEV), p.p_now.to(DEV), wl.offsets,
                  tri.TRI_KEYS_POST_ROPE, scores, ws)
    got = scores.cpu().numpy().astype(np.float64)
    for r, rec in enumerate(recs):
        bd = H.series_bound(wl.theta, cs[0], ms[0], r % Hh, wl.group, Kf[rec], wl.offsets)
        assert H.score_error(got[row_off[r]:row_off[r + 1]], ref[row_off[r]:row_off[r + 1]], bd) <= 1e-4
    # compact into a fresh table from the oracle's scores
    B, W = 256, 32
    ref32 = H.as_f32_exact(ref)
    ob = B // bs
    n_out = S * ob
    out_tbl = np.random.default_rng(3).permutation(n_out).reshape(S, ob).astype(np.int32)
    Ko = torch.zeros(1, n_out, bs, Hh, 128, dtype=torch.float8_e4m3fn, device=DEV)
    Vo = torch.zeros_like(Ko)
    kept = torch.full((S * Hh, B), -1, dtype=torch.int32, device=DEV)
    tri.tri_compact(m, kv, torch.tensor(ref32, dtype=torch.float32, device=DEV), B, W, Kd, Vd, None,
                    tri.out_paged(torch.as_tensor(out_tbl, device=DEV), bs, n_out), Ko, Vo, None, kept, None, ws)
    st, flags = tri.tri_status_check(ws)
    assert st == 0, flags
    Kob = H.raw_bits(Ko).reshape(-1, 128)
    kept = kept.cpu().numpy()
    for r, rec in enumerate(recs):
        s, h = r // Hh, r % Hh
        sel = oracle.select(ref32[row_off[r]:row_off[r + 1]], B, W)
        n = len(sel)
        np.testing.assert_array_equal(kept[r, :n], sel)
        i = np.arange(n)
        orec = (out_tbl[s, i // bs].astype(np.int64) * bs + i % bs) * Hh + h
        np.testing.assert_array_equal(Kob[orec], oracle.gather(Kb[rec], sel))


def test_fp8_full_size_sampled_rows():
    """The Qwen3-8B-shaped 32K cache in fp8, in the bench's launch configuration."""
    wl = synth.WORKLOADS["qwen3_8b_32k"]
    cache = synth.make_contig(wl, DEV)
    K8, V8 = synth.to_fp8(cache.K), synth.to_fp8(cache.V)
    del cache.K, cache.V
    L, S, Hh, B, W = wl.n_layers, 1, wl.n_kv_heads, wl.budget, wl.window
    rows = [5, 200]
    lays = sorted({cache.row_lhs(r)[0] for r in rows})
    c = torch.zeros(L, wl.n_q_heads, 64, 2, device=DEV)
    n = torch.ones(L, wl.n_q_heads, 64, device=DEV)
    cs = {}
    for li in lays:
        a, b = H.oracle_calibration(cache.qcal[li:li + 1])
        cs[li] = (H.as_f32_exact(a[0]), H.as_f32_exact(b[0]))
        c[li] = torch.tensor(cs[li][0], dtype=torch.float32, device=DEV)
        n[li] = torch.tensor(cs[li][1], dtype=torch.float32, device=DEV)
    m = tri.model(L, wl.n_q_heads, Hh, wl.theta)
    kv = tri.kv_contig(S, cache.row_off, cache.total, FP8)
    ws = tri.alloc_workspace(m, S, B)
    scores = torch.empty(cache.total, device=DEV)
    tri.tri_score(m, kv, K8, cache.pos, c, n, cache.p_now, wl.offsets, tri.TRI_KEYS_POST_ROPE, scores, ws)
    R = cache.n_rows
    Ko = torch.empty(R, B, 128, dtype=torch.float8_e4m3fn, device=DEV)
    Vo = torch.empty_like(Ko)
    kept = torch.empty(R, B, dtype=torch.int32, device=DEV)
    tri.tri_compact(m, kv, scores, B, W, K8, V8, None, tri.out_contig(), Ko, Vo, None, kept, None, ws)
    st, flags = tri.tri_status_check(ws)
    assert st == 0, flags
    sc = scores.cpu().numpy().astype(np.float64)
    kept = kept.cpu().numpy()
    for r in rows:
        li, s, h = cache.row_lhs(r)
        a, b = cache.row_off_np[r], cache.row_off_np[r + 1]
        Kf = H.to_f64(K8[a:b])
        ref = oracle.row_scores(wl.theta, cs[li][0], cs[li][1], h, wl.group, Kf,
                                cache.pos[a:b].cpu().numpy().astype(np.int64), True, int(cache.lens[s]),
                                wl.offsets, "collapsed")
        bd = H.series_bound(wl.theta, cs[li][0], cs[li][1], h, wl.group, Kf, wl.offsets)
        assert H.score_error(sc[a:b], ref, bd) <= 1e-4
        H.check_kept_within_ties(kept[r], ref, B, W, bd)
        assert np.array_equal(H.raw_bits(Ko[r]), H.raw_bits(K8[a:b])[kept[r]])
