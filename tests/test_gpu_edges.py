"""Limits and degenerate cases against the oracle: the most offsets
(TRI_MAX_OFFSETS), one query head per KV head and the most query heads per KV
head, paged block sizes at both ends of the allowed range, pre-RoPE positions
near the int32 limit, and budgets of a single key."""
import numpy as np
import pytest
import torch

import kv_cache_compression_calib_b200 as tri
import oracle
import synth
from tests import harness as H
from tests.test_gpu_parity import (POST, PRE, check_compaction_exact, gpu_compact, gpu_score, model_of,
                                   oracle_centres, oracle_scores, to_dev)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_most_offsets():
    offs = [1 + 3 * e for e in range(tri.TRI_MAX_OFFSETS - 2)] + [2 ** 20, 2 ** 30]
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="offs", batch=2, n_calib=32, n_offsets=1)
    host = synth.make_contig(wl, "cpu", lens=[900, 130])
    cs, ms = oracle_centres(host)
    dev = to_dev(host)
    m = model_of(wl, 1)
    kv = tri.kv_contig(2, dev.row_off, dev.total)
    ws = tri.alloc_workspace(m, 2, 64)
    scores = torch.empty(dev.total, device=DEV)
    tri.tri_score(m, kv, dev.K, dev.pos, torch.tensor(cs, dtype=torch.float32, device=DEV),
                  torch.tensor(ms, dtype=torch.float32, device=DEV), dev.p_now, offs, POST, scores, ws)
    got = scores.cpu().numpy().astype(np.float64)
    K = H.to_f64(host.K)
    pos = host.pos.numpy().astype(np.int64)
    for r in range(host.n_rows):
        li, s, h = host.row_lhs(r)
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        ref = oracle.row_scores(wl.theta, cs[li], ms[li], h, wl.group, K[a:b], pos[a:b], True, int(host.lens[s]),
                                offs, "literal")
        bd = H.series_bound(wl.theta, cs[li], ms[li], h, wl.group, K[a:b], offs)
        assert H.score_error(got[a:b], ref, bd) <= 1e-4
    with pytest.raises(tri.TriError):
        tri.tri_score(m, kv, dev.K, dev.pos, torch.tensor(cs, dtype=torch.float32, device=DEV),
                      torch.tensor(ms, dtype=torch.float32, device=DEV), dev.p_now, offs + [7], POST, scores, ws)


@pytest.mark.parametrize("hq,hkv", [(8, 8), (64, 4)])
def test_group_sizes(hq, hkv):
    wl = synth.WORKLOADS["single_layer_4k"].with_(name=f"g{hq}_{hkv}", n_q_heads=hq, n_kv_heads=hkv, batch=2,
                                                  n_calib=32)
    host = synth.make_contig(wl, "cpu", lens=[1500, 333])
    cs, ms = oracle_centres(host)
    ref, bound = oracle_scores(host, cs, ms, tier="collapsed")
    dev = to_dev(host)
    got = gpu_score(dev, cs, ms).cpu().numpy().astype(np.float64)
    assert H.score_error(got[:host.total], ref, bound) <= 1e-4
    ref32 = H.as_f32_exact(ref)
    res = gpu_compact(dev, torch.tensor(ref32, dtype=torch.float32, device=DEV), 256, 16)
    assert res["status"] == 0
    check_compaction_exact(host, res, ref32, 256, 16)


@pytest.mark.parametrize("bs", [1, 1024])
def test_paged_block_size_limits(bs):
    wl = synth.WORKLOADS["paged_16seq"].with_(name=f"bs{bs}", batch=2, n_calib=16, block_size=bs)
    lens = np.array([1500, 2100])
    p = synth.make_paged(wl, "cpu", lens=lens)
    qcal = synth.calib_queries(wl, 0, "cpu")[None]
    cs, ms = H.oracle_calibration(qcal)
    cs, ms = H.as_f32_exact(cs), H.as_f32_exact(ms)
    S, Hh = len(lens), wl.n_kv_heads
    row_off = synth.paged_row_offsets(lens, Hh)
    total = int(row_off[-1])
    Kf = H.to_f64(p.K).reshape(-1, 128)
    Kb = H.raw_bits(p.K).reshape(-1, 128)
    posf = p.pos.numpy().reshape(-1).astype(np.int64)
    m = model_of(wl, 1)
    kv = tri.kv_paged(S, torch.as_tensor(row_off, device=DEV), total, p.block_table.to(DEV), bs, p.K.shape[0])
    B, W = 1024, 64
    ws = tri.alloc_workspace(m, S, B)
    scores = torch.empty(total, device=DEV)
    Kd, Vd, pd = p.K.to(DEV), p.V.to(DEV), p.pos.to(DEV)
    tri.tri_score(m, kv, Kd, pd, torch.tensor(cs, dtype=torch.float32, device=DEV),
                  torch.tensor(ms, dtype=torch.float32, device=DEV), p.p_now.to(DEV), wl.offsets, POST, scores, ws)
    got = scores.cpu().numpy().astype(np.float64)
    ref = np.empty(total)
    recs = []
    for s in range(S):
        j = np.arange(int(lens[s]))
        blk = p.block_table_np[s, j // bs].astype(np.int64)
        for h in range(Hh):
            rec = (blk * bs + j % bs) * Hh + h
            recs.append(rec)
            r = s * Hh + h
            a, b = row_off[r], row_off[r + 1]
            ref[a:b] = oracle.row_scores(wl.theta, cs[0], ms[0], h, wl.group, Kf[rec], posf[rec], True, int(lens[s]),
                                         wl.offsets, "collapsed")
            bd = H.series_bound(wl.theta, cs[0], ms[0], h, wl.group, Kf[rec], wl.offsets)
            assert H.score_error(got[a:b], ref[a:b], bd) <= 1e-4
    ref32 = H.as_f32_exact(ref)
    ob = (B + bs - 1) // bs
    n_out = S * ob
    out_tbl = np.random.default_rng(2).permutation(n_out).reshape(S, ob).astype(np.int32)
    Ko = torch.zeros(1, n_out, bs, Hh, 128, dtype=torch.bfloat16, device=DEV)
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
        np.testing.assert_array_equal(kept[r, :len(sel)], sel)
        i = np.arange(len(sel))
        orec = (out_tbl[s, i // bs].astype(np.int64) * bs + i % bs) * Hh + h
        np.testing.assert_array_equal(Kob[orec], oracle.gather(Kb[rec], sel))


def test_pre_rope_positions_near_the_int32_limit():
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="far", batch=1, n_calib=32)
    host = synth.make_contig(wl, "cpu", lens=[700], rotate=False)
    shift = 2 ** 31 - 1 - 700 - 5000
    host.pos += shift
    host.p_now = host.p_now + shift + 4000  # the next position lies 4000 tokens past the last key
    cs, ms = oracle_centres(host)
    got = gpu_score(to_dev(host), cs, ms, key_mode=PRE).cpu().numpy().astype(np.float64)
    K = H.to_f64(host.K)
    pos = host.pos.numpy().astype(np.int64)
    p_now = int(host.p_now[0])
    for r in range(host.n_rows):
        li, s, h = host.row_lhs(r)
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        ref = oracle.row_scores(wl.theta, cs[li], ms[li], h, wl.group, K[a:b], pos[a:b], False, p_now, wl.offsets,
                                "collapsed")
        bd = H.series_bound(wl.theta, cs[li], ms[li], h, wl.group, K[a:b], wl.offsets)
        assert H.score_error(got[a:b], ref, bd) <= 1e-4


@pytest.mark.parametrize("B,W", [(1, 0), (1, 1), (2, 1)])
def test_single_key_budgets(B, W):
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="tiny", batch=3, n_calib=16)
    host = synth.make_contig(wl, "cpu", lens=[1, 2, 600])
    cs, ms = oracle_centres(host)
    ref, _ = oracle_scores(host, cs, ms, tier="collapsed")
    ref32 = H.as_f32_exact(ref)
    dev = to_dev(host)
    res = gpu_compact(dev, torch.tensor(ref32, dtype=torch.float32, device=DEV), B, W)
    assert res["status"] == 0
    check_compaction_exact(host, res, ref32, B, W)


@pytest.mark.parametrize("elem,mode", [("bf16", PRE), ("fp8", PRE), ("fp8", POST)])
def test_scores_with_a_total_not_a_multiple_of_four(elem, mode):
    """One KV head, rows of 1001, 2, 37, 0 and 5 keys (1045 in all): the last batch's
    final positions lie past the array's last whole 16-byte group, and rows shorter
    than a batch sit between longer ones."""
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="odd", n_q_heads=4, n_kv_heads=1, batch=5, n_calib=32)
    host = synth.make_contig(wl, "cpu", lens=[1001, 2, 37, 0, 5], rotate=(mode == POST))
    if elem == "fp8":
        host.K, host.V = synth.to_fp8(host.K), synth.to_fp8(host.V)
    assert host.total == 1045
    cs, ms = oracle_centres(host)
    dev = to_dev(host)
    got = gpu_score(dev, cs, ms, key_mode=mode).cpu().numpy().astype(np.float64)
    ref, bound = oracle_scores(host, cs, ms, post_rope=(mode == POST), tier="collapsed")
    assert H.score_error(got[:host.total], ref, bound) <= 1e-4
