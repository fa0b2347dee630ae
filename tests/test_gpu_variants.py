"""Head dims 64 and 256 and interleaved RoPE pairs (2f, 2f+1): calibration, scores,
selection and compaction on each layout against the oracle, in bf16 and fp8,
contiguous and paged.  Scores are checked against the collapsed oracle tier (pinned
equal to the literal triple sum for every layout) to 1e-4 of the series bound;
selection and compaction bit-exact on the oracle's fp32 scores."""
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
VARIANTS = [(64, "half"), (256, "half"), (128, "interleaved"), (64, "interleaved"), (256, "interleaved")]


def wl_of(d, style, **kw):
    base = synth.WORKLOADS["single_layer_4k"]
    return base.with_(name=f"d{d}_{style}", head_dim=d, rope_style=style, theta=1e6 if d == 128 else 1e4,
                      **kw)


@pytest.mark.parametrize("d,style", VARIANTS)
def test_variant_calibration(d, style):
    wl = wl_of(d, style, n_calib=257)
    q = synth.calib_queries(wl, 0, "cpu")[None]
    cs, ms = H.oracle_calibration(q, wl.interleaved)
    m = model_of(wl, 1)
    c = torch.empty(1, wl.n_q_heads, d // 2, 2, dtype=torch.float32, device=DEV)
    n = torch.empty(1, wl.n_q_heads, d // 2, dtype=torch.float32, device=DEV)
    tri.tri_calib(m, q.to(DEV).contiguous(), wl.n_calib, c, n)
    c, n = c.cpu().numpy().astype(np.float64), n.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(c - cs) <= 1e-6 * ms[..., None] + 1e-30)
    assert np.all(np.abs(n - ms) <= 1e-6 * ms)


@pytest.mark.parametrize("mode", [POST, PRE])
@pytest.mark.parametrize("d,style", VARIANTS)
def test_variant_scores_selection_gather(d, style, mode):
    wl = wl_of(d, style, batch=3, n_calib=96)
    host = synth.make_contig(wl, "cpu", lens=[4096, 1000, 37], rotate=(mode == POST))
    cs, ms = oracle_centres(host)
    ref, bound = oracle_scores(host, cs, ms, post_rope=(mode == POST), tier="collapsed")
    dev = to_dev(host)
    got = gpu_score(dev, cs, ms, key_mode=mode).cpu().numpy().astype(np.float64)
    assert H.score_error(got[:host.total], ref, bound) <= 1e-4
    ref32 = H.as_f32_exact(ref)
    B, W = 512, 64
    res = gpu_compact(dev, torch.tensor(ref32, dtype=torch.float32, device=DEV), B, W)
    assert res["status"] == 0, res["flags"]
    check_compaction_exact(host, res, ref32, B, W)


@pytest.mark.parametrize("d,style", [(64, "interleaved"), (256, "half"), (256, "interleaved")])
def test_variant_fp8(d, style):
    wl = wl_of(d, style, batch=2, n_calib=64)
    host = synth.make_contig(wl, "cpu", lens=[3000, 517])
    host.K = synth.to_fp8(host.K)
    host.V = synth.to_fp8(host.V)
    cs, ms = oracle_centres(host)
    ref, bound = oracle_scores(host, cs, ms, tier="collapsed")
    dev = to_dev(host)
    got = gpu_score(dev, cs, ms).cpu().numpy().astype(np.float64)
    assert H.score_error(got[:host.total], ref, bound) <= 1e-4
    ref32 = H.as_f32_exact(ref)
    B, W = 256, 16
    res = gpu_compact(dev, torch.tensor(ref32, dtype=torch.float32, device=DEV), B, W)
    assert res["status"] == 0, res["flags"]
    check_compaction_exact(host, res, ref32, B, W)


@pytest.mark.parametrize("d,style,elem", [(64, "half", "bf16"), (256, "interleaved", "bf16"),
                                          (256, "interleaved", "fp8")])
def test_variant_paged(d, style, elem):
    wl = synth.WORKLOADS["paged_16seq"].with_(name=f"paged_d{d}_{style}", batch=3, n_calib=64, head_dim=d,
                                              rope_style=style, theta=1e4)
    lens = np.array([300, 2100, 1024])
    p = synth.make_paged(wl, "cpu", lens=lens)
    if elem == "fp8":
        p.K = synth.to_fp8(p.K)
        p.V = synth.to_fp8(p.V)
    qcal = synth.calib_queries(wl, 0, "cpu")[None]
    cs, ms = H.oracle_calibration(qcal, wl.interleaved)
    cs, ms = H.as_f32_exact(cs), H.as_f32_exact(ms)
    S, Hh, bs = len(lens), wl.n_kv_heads, wl.block_size
    row_off = synth.paged_row_offsets(lens, Hh)
    total = int(row_off[-1])
    Kf = H.to_f64(p.K).reshape(-1, d)
    Kb = H.raw_bits(p.K).reshape(-1, d)
    Vb = H.raw_bits(p.V).reshape(-1, d)
    posf = p.pos.numpy().reshape(-1)
    recs = []
    ref = np.empty(total)
    bound = np.empty(total)
    for s in range(S):
        j = np.arange(int(lens[s]))
        blk = p.block_table_np[s, j // bs].astype(np.int64)
        for h in range(Hh):
            rec = (blk * bs + j % bs) * Hh + h
            recs.append(rec)
            r = s * Hh + h
            a, b = row_off[r], row_off[r + 1]
            ref[a:b] = oracle.row_scores(wl.theta, cs[0], ms[0], h, wl.group, Kf[rec], posf[rec].astype(np.int64),
                                         True, int(lens[s]), wl.offsets, "collapsed", wl.interleaved)
            bound[a:b] = H.series_bound(wl.theta, cs[0], ms[0], h, wl.group, Kf[rec], wl.offsets, wl.interleaved)
    m = model_of(wl, 1)
    kv = tri.kv_paged(S, torch.as_tensor(row_off, device=DEV), total, p.block_table.to(DEV), bs, p.K.shape[0],
                      tri.elem_type_of(p.K))
    B, W = 256, 32
    ws = tri.alloc_workspace(m, S, B)
    scores = torch.empty(total, device=DEV)
    Kd, Vd, pd = p.K.to(DEV), p.V.to(DEV), p.pos.to(DEV)
    tri.tri_score(m, kv, Kd, pd, torch.tensor(cs, dtype=torch.float32, device=DEV),
                  torch.tensor(ms, dtype=torch.float32, device=DEV), p.p_now.to(DEV), wl.offsets,
                  tri.TRI_KEYS_POST_ROPE, scores, ws)
    got = scores.cpu().numpy().astype(np.float64)
    assert H.score_error(got, ref, bound) <= 1e-4
    ref32 = H.as_f32_exact(ref)
    ob = (B + bs - 1) // bs
    n_out = S * ob
    out_tbl = np.random.default_rng(5).permutation(n_out).reshape(S, ob).astype(np.int32)
    Ko = torch.zeros(1, n_out, bs, Hh, d, dtype=p.K.dtype, device=DEV)
    Vo = torch.zeros_like(Ko)
    po = torch.full((1, n_out, bs, Hh), -1, dtype=torch.int32, device=DEV)
    kept = torch.full((S * Hh, B), -1, dtype=torch.int32, device=DEV)
    tri.tri_compact(m, kv, torch.tensor(ref32, dtype=torch.float32, device=DEV), B, W, Kd, Vd, pd,
                    tri.out_paged(torch.as_tensor(out_tbl, device=DEV), bs, n_out), Ko, Vo, po, kept, None, ws)
    st, flags = tri.tri_status_check(ws)
    assert st == 0, flags
    Kob = H.raw_bits(Ko).reshape(-1, d)
    Vob = H.raw_bits(Vo).reshape(-1, d)
    pob = po.cpu().numpy().reshape(-1)
    kept = kept.cpu().numpy()
    for r, rec in enumerate(recs):
        s, h = r // Hh, r % Hh
        sel = oracle.select(ref32[row_off[r]:row_off[r + 1]], B, W)
        n = len(sel)
        np.testing.assert_array_equal(kept[r, :n], sel)
        i = np.arange(n)
        orec = (out_tbl[s, i // bs].astype(np.int64) * bs + i % bs) * Hh + h
        np.testing.assert_array_equal(Kob[orec], oracle.gather(Kb[rec], sel))
        np.testing.assert_array_equal(Vob[orec], oracle.gather(Vb[rec], sel))
        np.testing.assert_array_equal(pob[orec], oracle.gather(posf[rec], sel))
