"""Full-size workloads, in the launch configuration bench.py times, checked on
sampled rows against the oracle and by properties on every row.

Per sampled row: scores within 1e-4 of the series bound (oracle, collapsed
tier); selection end to end within boundary ties; selection bit-exact when
the row's scores are replaced by the oracle's fp32 scores; compacted records
bit-exact against the oracle's gather.  Every row: kept count, ascending
order, the window kept, and (on the GPU's own scores) min kept score >= max
evicted score.
"""
import gc

import numpy as np
import pytest
import torch

import kv_cache_compression_calib_b200 as tri
import oracle
import synth
from tests import harness as H

pytestmark = pytest.mark.gpu
DEV = "cuda"


def free_gib():
    f, _ = torch.cuda.mem_get_info()
    return f / 2 ** 30


def calibrate_layers(cache, layers_for_oracle):
    """fp32 centres for every layer: the oracle's for `layers_for_oracle`, the others
    from tri_calib (those layers' rows are only property-checked)."""
    wl = cache.wl
    L = len(cache.layers)
    m = tri.model(L, wl.n_q_heads, wl.n_kv_heads, wl.theta)
    c = torch.empty(L, wl.n_q_heads, 64, 2, device=DEV)
    n = torch.empty(L, wl.n_q_heads, 64, device=DEV)
    tri.tri_calib(m, cache.qcal, wl.n_calib, c, n)
    cs = {}
    for li in sorted(set(layers_for_oracle)):
        a, b = H.oracle_calibration(cache.qcal[li:li + 1])
        cs[li] = (H.as_f32_exact(a[0]), H.as_f32_exact(b[0]))
        c[li] = torch.tensor(cs[li][0], dtype=torch.float32, device=DEV)
        n[li] = torch.tensor(cs[li][1], dtype=torch.float32, device=DEV)
    return m, c, n, cs


def run_contig(cache, m, c, n, B, W, scores=None):
    S = len(cache.lens)
    R, total = cache.n_rows, cache.total
    kv = tri.kv_contig(S, cache.row_off, total)
    ws = tri.alloc_workspace(m, S, B)
    if scores is None:
        scores = torch.empty(total, dtype=torch.float32, device=DEV)
        tri.tri_score(m, kv, cache.K, cache.pos, c, n, cache.p_now, cache.wl.offsets,
                      tri.TRI_KEYS_POST_ROPE, scores, ws)
    Ko = torch.empty(R, B, 128, dtype=torch.bfloat16, device=DEV)
    Vo = torch.empty_like(Ko)
    po = torch.empty(R, B, dtype=torch.int32, device=DEV)
    kept = torch.full((R, B), -1, dtype=torch.int32, device=DEV)
    cnt = torch.empty(R, dtype=torch.int32, device=DEV)
    tri.tri_compact(m, kv, scores, B, W, cache.K, cache.V, cache.pos, tri.out_contig(), Ko, Vo, po,
                    kept, cnt, ws)
    st, flags = tri.tri_status_check(ws)
    assert st == 0, flags
    return scores, Ko, Vo, po, kept, cnt


def check_all_rows(cache, scores, kept, cnt, B, W):
    """Properties of every row, on the GPU's own fp32 scores."""
    sc = scores.cpu().numpy()
    kept = kept.cpu().numpy()
    cnt = cnt.cpu().numpy()
    for r in range(cache.n_rows):
        a, b = cache.row_off_np[r], cache.row_off_np[r + 1]
        N = b - a
        k = kept[r, :cnt[r]]
        assert cnt[r] == min(N, B)
        assert np.all(np.diff(k) > 0) and k[0] >= 0 and k[-1] < N
        if N > B:
            assert np.all(k[-W:] == np.arange(N - W, N)) if W else True
            s = sc[a:b]
            mask = np.zeros(N, bool)
            mask[k] = True
            mask[N - W:] = False
            ev = np.ones(N, bool)
            ev[k] = False
            if ev.any():
                assert s[mask].min() >= s[ev].max()


def check_sampled_rows(cache, cs, rows, scores, kept, Ko, Vo, po, B, W):
    wl = cache.wl
    sc = scores.cpu().numpy().astype(np.float64)
    kept = kept.cpu().numpy()
    worst = 0.0
    refs = {}
    for r in rows:
        li, s, h = cache.row_lhs(r)
        a, b = cache.row_off_np[r], cache.row_off_np[r + 1]
        Kb = H.bits16(cache.K[a:b])
        Kf = oracle.bf16_bits_to_f64(Kb)
        pos = cache.pos[a:b].cpu().numpy().astype(np.int64)
        c0, m0 = cs[li]
        ref = oracle.row_scores(wl.theta, c0, m0, h, wl.group, Kf, pos, True, int(cache.lens[s]),
                                wl.offsets, "collapsed")
        bd = H.series_bound(wl.theta, c0, m0, h, wl.group, Kf, wl.offsets)
        worst = max(worst, H.score_error(sc[a:b], ref, bd))
        n = min(b - a, B)
        H.check_kept_within_ties(kept[r, :n], ref, B, W, bd)
        assert np.array_equal(H.bits16(Ko[r, :n]), Kb[kept[r, :n]])
        refs[r] = ref
    assert worst <= 1e-4, worst
    return refs


def check_exact_given_oracle_scores(cache, m, c, n, scores, refs, B, W):
    """Overwrite the sampled rows' scores with the oracle's fp32 scores and compact
    again: those rows must then match oracle.select / oracle.gather bit for bit."""
    sc = scores.clone()
    for r, ref in refs.items():
        a, b = cache.row_off_np[r], cache.row_off_np[r + 1]
        sc[a:b] = torch.tensor(ref, dtype=torch.float32, device=DEV)
    _, Ko, Vo, po, kept, cnt = run_contig(cache, m, c, n, B, W, scores=sc)
    kept = kept.cpu().numpy()
    for r, ref in refs.items():
        a, b = cache.row_off_np[r], cache.row_off_np[r + 1]
        sel = oracle.select(H.as_f32_exact(ref), B, W)
        k = len(sel)
        np.testing.assert_array_equal(kept[r, :k], sel)
        np.testing.assert_array_equal(H.bits16(Ko[r, :k]), oracle.gather(H.bits16(cache.K[a:b]), sel))
        np.testing.assert_array_equal(H.bits16(Vo[r, :k]), oracle.gather(H.bits16(cache.V[a:b]), sel))
        np.testing.assert_array_equal(po[r, :k].cpu().numpy(),
                                      oracle.gather(cache.pos[a:b].cpu().numpy(), sel))


def full_contig_case(wl, rows, B=None, layers=None):
    B = B or wl.budget
    cache = synth.make_contig(wl, DEV, layers=layers)
    lay = sorted({cache.row_lhs(r)[0] for r in rows})
    m, c, n, cs = calibrate_layers(cache, lay)
    scores, Ko, Vo, po, kept, cnt = run_contig(cache, m, c, n, B, wl.window)
    check_all_rows(cache, scores, kept, cnt, B, wl.window)
    refs = check_sampled_rows(cache, cs, rows, scores, kept, Ko, Vo, po, B, wl.window)
    del Ko, Vo, po, kept, cnt
    check_exact_given_oracle_scores(cache, m, c, n, scores, refs, B, wl.window)
    return cache


def test_qwen3_8b_32k_full():
    wl = synth.WORKLOADS["qwen3_8b_32k"]
    full_contig_case(wl, rows=[0, 77, 150, 287])


def test_sweep_b64_one_layer_each_budget():
    wl = synth.WORKLOADS["sweep_b64"]
    lens = wl.seq_lengths()
    order = np.argsort(lens)
    for B in synth.SWEEP_BUDGETS:
        # shortest, longest and a middle sequence, different heads
        rows = [int(order[0]) * 8 + 1, int(order[-1]) * 8 + 6, int(order[32]) * 8 + 3]
        full_contig_case(wl, rows=rows, B=B, layers=[5])
        gc.collect()
        torch.cuda.empty_cache()


def test_sweep_adversarial_zero_centre_layer():
    wl = synth.WORKLOADS["sweep_b64_adversarial"]
    z = wl.zero_centre_pairs()
    layer = int(np.nonzero(z.any(axis=1))[0][0])
    hz = int(np.nonzero(z[layer])[0][0])
    hn = int(np.nonzero(~z[layer])[0][0])
    rows = [0 * 8 + hz, 17 * 8 + hz, 40 * 8 + hn]
    full_contig_case(wl, rows=rows, layers=[layer])


@pytest.mark.skipif(not torch.cuda.is_available() or
                    torch.cuda.get_device_properties(0).total_memory < 170 * 2 ** 30,
                    reason="needs a 180 GB device")
def test_qwen3_32b_128k_full():
    wl = synth.WORKLOADS["qwen3_32b_128k"]
    gc.collect()
    torch.cuda.empty_cache()
    full_contig_case(wl, rows=[0, 1029, 2047])


# ------------------------------------------------------ paged re-score rounds

def test_paged_16seq_rounds():
    """16 sequences of 8K..32K keys in 16-token blocks: compact the prefill to
    B = 2048, then 8 rounds of +128 decode tokens, each merged with the retained
    2048 and re-scored, compacted into a fresh shuffled block table.  Sampled rows
    keep an oracle-side mirror built only from generator bits and oracle
    selections; each round's GPU input for those rows is checked equal to it."""
    wl = synth.WORKLOADS["paged_16seq"]
    B, W, bs, Hh = wl.budget, wl.window, wl.block_size, wl.n_kv_heads
    lens = wl.seq_lengths()
    S = len(lens)
    pg = synth.make_paged(wl, DEV, lens=lens)
    m, c, n, _ = None, None, None, None
    qcal = synth.calib_queries(wl, 0, DEV)[None]
    cs, ms = H.oracle_calibration(qcal)
    cs, ms = H.as_f32_exact(cs), H.as_f32_exact(ms)
    c = torch.tensor(cs, dtype=torch.float32, device=DEV)
    n = torch.tensor(ms, dtype=torch.float32, device=DEV)
    m = tri.model(1, wl.n_q_heads, Hh, wl.theta)
    rows = [s * Hh + (s % Hh) for s in range(S)]  # one head per sequence

    def recs_of(table, s, h, count):
        j = np.arange(count)
        return (table[s, j // bs].astype(np.int64) * bs + j % bs) * Hh + h

    # oracle mirror of sampled rows: generator bits
    Kh = H.bits16(pg.K).reshape(-1, 128)
    Vh = H.bits16(pg.V).reshape(-1, 128)
    Ph = pg.pos.cpu().numpy().reshape(-1)
    mirror = {}
    for r in rows:
        s, h = r // Hh, r % Hh
        rec = recs_of(pg.block_table_np, s, h, int(lens[s]))
        mirror[r] = (Kh[rec], Vh[rec], Ph[rec].astype(np.int64))

    K_in, V_in, P_in, tbl_in = pg.K, pg.V, pg.pos, pg.block_table
    n_blocks_in = pg.K.shape[0]
    cur = lens.copy()
    p_now = lens.copy()
    ob = (B + wl.rescore_every + bs - 1) // bs  # room for the retained keys + one round of tokens
    n_out = S * ob
    rng = np.random.default_rng(77)
    for rnd in range(wl.rounds + 1):
        row_off = synth.paged_row_offsets(cur, Hh)
        total = int(row_off[-1])
        ro = torch.as_tensor(row_off, device=DEV)
        kv = tri.kv_paged(S, ro, total, tbl_in, bs, n_blocks_in)
        ws = tri.alloc_workspace(m, S, B)
        pn = torch.as_tensor(p_now, device=DEV)
        scores = torch.empty(total, dtype=torch.float32, device=DEV)
        tri.tri_score(m, kv, K_in, P_in, c, n, pn, wl.offsets, tri.TRI_KEYS_POST_ROPE, scores, ws)
        # the GPU's inputs for sampled rows equal the oracle mirror
        tin = tbl_in.cpu().numpy()
        Kin = H.bits16(K_in).reshape(-1, 128)
        sc = scores.cpu().numpy().astype(np.float64)
        sc_exact = scores.clone()
        refs = {}
        for r in rows:
            s, h = r // Hh, r % Hh
            rec = recs_of(tin, s, h, int(cur[s]))
            assert np.array_equal(Kin[rec], mirror[r][0])
            Kf = oracle.bf16_bits_to_f64(mirror[r][0])
            ref = oracle.row_scores(wl.theta, cs[0], ms[0], h, wl.group, Kf, mirror[r][2], True,
                                    int(p_now[s]), wl.offsets, "collapsed")
            bd = H.series_bound(wl.theta, cs[0], ms[0], h, wl.group, Kf, wl.offsets)
            a, b = row_off[r], row_off[r + 1]
            assert H.score_error(sc[a:b], ref, bd) <= 1e-4, (rnd, r)
            refs[r] = (ref, bd)
            sc_exact[a:b] = torch.tensor(ref, dtype=torch.float32, device=DEV)
        # (1) end to end on the GPU's scores, (2) exact on the oracle's for sampled rows
        out_tbl = rng.permutation(n_out).reshape(S, ob).astype(np.int32)
        otd = torch.as_tensor(out_tbl, device=DEV)
        outs = []
        for sco in (scores, sc_exact):
            Ko = torch.zeros(1, n_out, bs, Hh, 128, dtype=torch.bfloat16, device=DEV)
            Vo = torch.zeros_like(Ko)
            Po = torch.full((1, n_out, bs, Hh), -1, dtype=torch.int32, device=DEV)
            kept = torch.full((S * Hh, B), -1, dtype=torch.int32, device=DEV)
            tri.tri_compact(m, kv, sco, B, W, K_in, V_in, P_in, tri.out_paged(otd, bs, n_out), Ko, Vo,
                            Po, kept, None, ws)
            st, flags = tri.tri_status_check(ws)
            assert st == 0, flags
            outs.append((Ko, Vo, Po, kept.cpu().numpy()))
        kept_gpu = outs[0][3]
        Ko, Vo, Po, kept_ex = outs[1]
        Kob = H.bits16(Ko).reshape(-1, 128)
        Vob = H.bits16(Vo).reshape(-1, 128)
        Pob = Po.cpu().numpy().reshape(-1)
        for r in rows:
            s, h = r // Hh, r % Hh
            ref, bd = refs[r]
            k = min(int(cur[s]), B)
            H.check_kept_within_ties(kept_gpu[r, :k], ref, B, W, bd)
            sel = oracle.select(H.as_f32_exact(ref), B, W)
            np.testing.assert_array_equal(kept_ex[r, :k], sel)
            orec = recs_of(out_tbl, s, h, k)
            newK = oracle.gather(mirror[r][0], sel)
            newV = oracle.gather(mirror[r][1], sel)
            newP = oracle.gather(mirror[r][2], sel)
            assert np.array_equal(Kob[orec], newK) and np.array_equal(Vob[orec], newV)
            assert np.array_equal(Pob[orec], newP)
            mirror[r] = (newK, newV, newP)
        cur = np.minimum(cur, B)
        if rnd == wl.rounds:
            break
        # decode 128 tokens per sequence into the fresh table, after the retained keys
        Kn, Vn = synth.decode_keys(wl, 0, rnd, p_now, wl.rescore_every, DEV)
        for s in range(S):
            j = np.arange(int(cur[s]), int(cur[s]) + wl.rescore_every)
            blk = torch.as_tensor(out_tbl[s, j // bs].astype(np.int64), device=DEV)
            slot = torch.as_tensor(j % bs, device=DEV)
            Ko[0, blk, slot] = Kn[s]
            Vo[0, blk, slot] = Vn[s]
            Po[0, blk, slot] = torch.arange(int(p_now[s]), int(p_now[s]) + wl.rescore_every,
                                            device=DEV, dtype=torch.int32)[:, None]
        Knh, Vnh = H.bits16(Kn), H.bits16(Vn)
        for r in rows:
            s, h = r // Hh, r % Hh
            pnew = np.arange(int(p_now[s]), int(p_now[s]) + wl.rescore_every, dtype=np.int64)
            mirror[r] = (np.concatenate([mirror[r][0], Knh[s, :, h]]),
                         np.concatenate([mirror[r][1], Vnh[s, :, h]]),
                         np.concatenate([mirror[r][2], pnew]))
        cur = cur + wl.rescore_every
        p_now = p_now + wl.rescore_every
        K_in, V_in, P_in, tbl_in, n_blocks_in = Ko, Vo, Po, otd, n_out
