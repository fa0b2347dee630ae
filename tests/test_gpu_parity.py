"""GPU parity against the CPU oracle on sizes the oracle finishes in seconds.

Scores: |S_gpu - S_oracle| <= 1e-4 * M_j, M_j = sum_f (|A_f| + |c_f|)|k_f| the
absolute-value bound of the row's series (fp32 accumulation of up to 192
terms of size <= M_j keeps the error near 1e-6 M_j; 1e-4 is the stated bar).
Selection given identical fp32 scores: bit-exact.  Selection end to end: equal
except at ties within 1e-5 of the oracle's threshold.  Compaction given the
index set: bit-exact.  All calls go through the C ABI (libtri.so).
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_calib_b200 as tri
import oracle
import synth
from tests import harness as H

pytestmark = pytest.mark.gpu
DEV = "cuda"
POST, PRE = tri.TRI_KEYS_POST_ROPE, tri.TRI_KEYS_PRE_ROPE


def model_of(wl, n_layers):
    style = tri.TRI_ROPE_INTERLEAVED if wl.interleaved else tri.TRI_ROPE_HALF
    return tri.model(n_layers, wl.n_q_heads, wl.n_kv_heads, wl.theta, head_dim=wl.head_dim, rope_style=style)


def to_dev(cache: synth.ContigCache) -> synth.ContigCache:
    """Copy a host-generated cache to the GPU (same bits)."""
    c = synth.ContigCache(cache.wl, cache.layers, cache.lens, cache.K.to(DEV),
                          cache.V.to(DEV) if cache.V is not None else None, cache.pos.to(DEV),
                          cache.row_off.to(DEV), cache.row_off_np, cache.p_now.to(DEV),
                          cache.qcal.to(DEV))
    return c


def oracle_centres(cache):
    cs, ms = H.oracle_calibration(cache.qcal, cache.wl.interleaved)
    return H.as_f32_exact(cs), H.as_f32_exact(ms)


def oracle_scores(cache, cs, ms, post_rope=True, tier="literal", rows=None):
    wl = cache.wl
    K = H.to_f64(cache.K)
    pos = cache.pos.cpu().numpy().astype(np.int64)
    out = np.full(cache.total, np.nan)
    bounds = np.full(cache.total, np.nan)
    rows = range(cache.n_rows) if rows is None else rows
    for r in rows:
        li, s, h = cache.row_lhs(r)
        a, b = cache.row_off_np[r], cache.row_off_np[r + 1]
        if b == a:
            continue
        out[a:b] = oracle.row_scores(wl.theta, cs[li], ms[li], h, wl.group, K[a:b], pos[a:b],
                                     post_rope, int(cache.lens[s]), wl.offsets, tier, wl.interleaved)
        bounds[a:b] = H.series_bound(wl.theta, cs[li], ms[li], h, wl.group, K[a:b], wl.offsets,
                                     wl.interleaved)
    return out, bounds


def gpu_score(cache, cs, ms, key_mode=POST, B=1):
    wl = cache.wl
    m = model_of(wl, len(cache.layers))
    S = len(cache.lens)
    kv = tri.kv_contig(S, cache.row_off, cache.total, tri.elem_type_of(cache.K))
    c32 = torch.tensor(cs, dtype=torch.float32, device=DEV)
    m32 = torch.tensor(ms, dtype=torch.float32, device=DEV)
    ws = tri.alloc_workspace(m, S, B)
    scores = torch.full((max(cache.total, 1),), float("nan"), dtype=torch.float32, device=DEV)
    tri.tri_score(m, kv, cache.K, cache.pos, c32, m32, cache.p_now, wl.offsets, key_mode, scores, ws)
    st, flags = tri.tri_status_check(ws)
    assert st == 0 and flags == 0
    return scores


def gpu_compact(cache, scores, B, W):
    wl = cache.wl
    m = model_of(wl, len(cache.layers))
    S = len(cache.lens)
    R = cache.n_rows
    kv = tri.kv_contig(S, cache.row_off, cache.total, tri.elem_type_of(cache.K))
    ws = tri.alloc_workspace(m, S, B)
    Ko = torch.zeros(R, B, wl.head_dim, dtype=cache.K.dtype, device=DEV)
    Vo = torch.zeros(R, B, wl.head_dim, dtype=cache.K.dtype, device=DEV)
    po = torch.full((R, B), -7, dtype=torch.int32, device=DEV)
    kept = torch.full((R, B), -1, dtype=torch.int32, device=DEV)
    cnt = torch.full((R,), -1, dtype=torch.int32, device=DEV)
    tri.tri_compact(m, kv, scores, B, W, cache.K, cache.V, cache.pos, tri.out_contig(), Ko, Vo, po,
                    kept, cnt, ws)
    st, flags = tri.tri_status_check(ws)
    return dict(K=Ko.cpu(), V=Vo.cpu(), pos=po.cpu(), kept=kept.cpu().numpy(), cnt=cnt.cpu().numpy(),
                status=st, flags=flags)


def check_compaction_exact(cache, res, ref_scores32, B, W):
    """Kept sets == oracle.select of the same fp32 scores; K/V/pos == oracle.gather."""
    Kb, Vb = H.raw_bits(cache.K), H.raw_bits(cache.V)
    pos = cache.pos.cpu().numpy()
    Kob, Vob = H.raw_bits(res["K"]), H.raw_bits(res["V"])
    for r in range(cache.n_rows):
        a, b = cache.row_off_np[r], cache.row_off_np[r + 1]
        ref = oracle.select(ref_scores32[a:b], B, W)
        n = len(ref)
        assert res["cnt"][r] == n
        np.testing.assert_array_equal(res["kept"][r, :n], ref, err_msg=f"row {r}")
        np.testing.assert_array_equal(Kob[r, :n], oracle.gather(Kb[a:b], ref))
        np.testing.assert_array_equal(Vob[r, :n], oracle.gather(Vb[a:b], ref))
        np.testing.assert_array_equal(res["pos"][r, :n].numpy(), oracle.gather(pos[a:b], ref))
        assert np.all(res["kept"][r, n:] == -1)  # nothing written past the count


# ------------------------------------------------------------------ calib

def test_calibration_matches_oracle():
    wl = synth.WORKLOADS["single_layer_4k"]
    for nq in (1, 3, 1024):
        w = wl.with_(n_calib=nq)
        q = synth.calib_queries(w, 0, "cpu")[None]
        cs, ms = H.oracle_calibration(q)
        m = model_of(w, 1)
        c = torch.empty(1, 32, 64, 2, dtype=torch.float32, device=DEV)
        n = torch.empty(1, 32, 64, dtype=torch.float32, device=DEV)
        tri.tri_calib(m, q.to(DEV).contiguous(), nq, c, n)
        c, n = c.cpu().numpy().astype(np.float64), n.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(c - cs) <= 1e-6 * ms[..., None] + 1e-30)
        assert np.all(np.abs(n - ms) <= 1e-6 * ms)
        if nq == 1:
            np.testing.assert_allclose(n, np.hypot(cs[..., 0], cs[..., 1]), rtol=1e-6)


# ------------------------------------------------------- single-layer 4K

@pytest.fixture(scope="module")
def cfg1():
    wl = synth.WORKLOADS["single_layer_4k"]
    host = synth.make_contig(wl, "cpu")
    cs, ms = oracle_centres(host)
    ref, bound = oracle_scores(host, cs, ms, post_rope=True, tier="literal")
    return wl, host, to_dev(host), cs, ms, ref, bound


def test_cfg1_scores_match_literal_oracle(cfg1):
    wl, host, dev, cs, ms, ref, bound = cfg1
    got = gpu_score(dev, cs, ms).cpu().numpy().astype(np.float64)
    err = H.score_error(got, ref, bound)
    assert err <= 1e-4, err
    big = np.abs(ref) > 0.1 * bound
    assert np.max(np.abs(got - ref)[big] / np.abs(ref[big])) <= 1e-4


def test_cfg1_selection_and_gather_bit_exact(cfg1):
    wl, host, dev, cs, ms, ref, bound = cfg1
    ref32 = H.as_f32_exact(ref)
    res = gpu_compact(dev, torch.tensor(ref32, dtype=torch.float32, device=DEV), wl.budget,
                      wl.window)
    assert res["status"] == 0
    check_compaction_exact(host, res, ref32, wl.budget, wl.window)


def test_cfg1_end_to_end(cfg1):
    wl, host, dev, cs, ms, ref, bound = cfg1
    scores = gpu_score(dev, cs, ms)
    res = gpu_compact(dev, scores, wl.budget, wl.window)
    assert res["status"] == 0
    Kb = H.bits16(host.K)
    Kob = res["K"].view(torch.int16).numpy()
    for r in range(host.n_rows):
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        kept = res["kept"][r, :wl.budget]
        H.check_kept_within_ties(kept, ref[a:b], wl.budget, wl.window, bound[a:b])
        # each output record is the input record at the slot reported
        assert np.array_equal(Kob[r], Kb[a:b][kept])


# -------------------------------------------------------- ragged / edges

RAGGED_LENS = [0, 1, 7, 15, 16, 17, 33, 63, 64, 65, 100, 513, 1000, 2049]


@pytest.fixture(scope="module")
def ragged():
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="ragged", n_layers=2, batch=len(RAGGED_LENS),
                                                   n_calib=64)
    host = synth.make_contig(wl, "cpu", lens=RAGGED_LENS)
    cs, ms = oracle_centres(host)
    ref, bound = oracle_scores(host, cs, ms, tier="literal")
    return wl, host, to_dev(host), cs, ms, ref, bound


def test_ragged_scores(ragged):
    wl, host, dev, cs, ms, ref, bound = ragged
    got = gpu_score(dev, cs, ms).cpu().numpy().astype(np.float64)[:host.total]
    assert H.score_error(got, ref, bound) <= 1e-4


@pytest.mark.parametrize("B,W", [(64, 16), (1, 0), (1, 1), (16, 16), (100, 0), (512, 64), (17, 3)])
def test_ragged_selection_and_gather_bit_exact(ragged, B, W):
    wl, host, dev, cs, ms, ref, bound = ragged
    ref32 = H.as_f32_exact(ref)
    res = gpu_compact(dev, torch.tensor(ref32, dtype=torch.float32, device=DEV), B, W)
    assert res["status"] == 0
    check_compaction_exact(host, res, ref32, B, W)


def test_ragged_end_to_end(ragged):
    wl, host, dev, cs, ms, ref, bound = ragged
    scores = gpu_score(dev, cs, ms)
    res = gpu_compact(dev, scores, 64, 16)
    for r in range(host.n_rows):
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        H.check_kept_within_ties(res["kept"][r, :res["cnt"][r]], ref[a:b], 64, 16, bound[a:b])


# --------------------------------------------------- ties, NaN, signed 0

def _scores_case(kind, n, rng):
    if kind == "all_equal":
        return np.full(n, 2.5)
    if kind == "quantized":
        return np.round(rng.standard_normal(n) * 3)
    if kind == "signed_zero":
        s = np.where(rng.random(n) < 0.5, -0.0, 0.0)
        s[rng.random(n) < 0.1] = 1.0
        return s
    if kind == "nan":
        s = rng.standard_normal(n)
        s[rng.random(n) < 0.05] = np.nan
        return s
    if kind == "wide":
        return rng.standard_normal(n) * np.exp(rng.standard_normal(n) * 20)
    if kind == "subnormal":
        return rng.standard_normal(n) * 1e-42
    if kind == "huge":
        s = rng.standard_normal(n)
        s[::5] = 3.0e38
        s[1::7] = -3.0e38
        return s
    if kind == "straddle":
        return rng.standard_normal(n) * 50 + 10
    if kind == "outlier":
        s = rng.standard_normal(n)
        s[::1000] = 1e6
        return s
    if kind == "inf":
        s = rng.standard_normal(n)
        s[::97] = np.inf
        s[::89] = -np.inf
        return s
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["all_equal", "quantized", "signed_zero", "nan", "wide", "inf",
                                  "subnormal", "huge", "straddle", "outlier"])
def test_selection_special_scores(ragged, kind):
    wl, host, dev, cs, ms, ref, bound = ragged
    rng = np.random.default_rng(5)
    s32 = H.as_f32_exact(_scores_case(kind, host.total, rng))
    res = gpu_compact(dev, torch.tensor(s32, dtype=torch.float32, device=DEV), 64, 16)
    check_compaction_exact(host, res, s32, 64, 16)
    if kind == "nan":
        assert res["flags"] & tri.TRI_FLAG_NONFINITE
    else:
        assert res["status"] == 0


# ----------------------------------------------------------- pre-RoPE keys

def test_pre_rope_keys_match_literal_oracle():
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="pre", batch=2, seq_len=(3000, 4500),
                                                   n_calib=128)
    host = synth.make_contig(wl, "cpu", rotate=False)
    cs, ms = oracle_centres(host)
    ref, bound = oracle_scores(host, cs, ms, post_rope=False, tier="literal")
    got = gpu_score(to_dev(host), cs, ms, key_mode=PRE).cpu().numpy().astype(np.float64)
    assert H.score_error(got, ref, bound) <= 1e-4


def test_pre_rope_shifted_positions():
    """Positions far from 0 (p_now ~ 1.3e5): the fixed-point phase keeps fp32 exact enough."""
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="preshift", n_calib=64)
    host = synth.make_contig(wl, "cpu", rotate=False)
    shift = 127000
    host.pos += shift
    host.p_now = host.p_now + shift
    cs, ms = oracle_centres(host)
    K = H.to_f64(host.K)
    pos = host.pos.numpy().astype(np.int64)
    dev = to_dev(host)
    got = gpu_score(dev, cs, ms, key_mode=PRE).cpu().numpy().astype(np.float64)
    for r in (0, 7):
        li, s, h = host.row_lhs(r)
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        ref = oracle.row_scores(wl.theta, cs[li], ms[li], h, wl.group, K[a:b], pos[a:b], False,
                                int(host.p_now[s]), wl.offsets, "collapsed")
        bd = H.series_bound(wl.theta, cs[li], ms[li], h, wl.group, K[a:b], wl.offsets)
        assert H.score_error(got[a:b], ref, bd) <= 1e-4


def irregular_positions(n, r):
    """Position patterns per row that break the regular stride: gaps (a compacted
    cache), a descending run, repeats, a run across the end of the int32 range,
    and runs of 16 with gaps between them."""
    rng = np.random.default_rng(1000 + r)
    kind = r % 5
    if kind == 0:
        return np.sort(rng.choice(50000, n, replace=False))
    if kind == 1:
        return np.arange(n)[::-1].copy()
    if kind == 2:
        return np.arange(n) // 2
    if kind == 3:
        top = np.iinfo(np.int32).max
        return np.concatenate([np.arange(top - n // 2 + 1, top + 1), np.iinfo(np.int32).min + np.arange(n - n // 2)])
    return (np.arange(n) // 16) * 100 + np.arange(n) % 16


def test_pre_rope_irregular_positions():
    """The pre-RoPE kernels chain a lane's rotated coefficients only where a key sits
    exactly NG positions after the last one; every other key (gaps, descending or
    repeated positions, a run across the int32 range's end) takes its own phase."""
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="preirr", n_calib=64)
    host = synth.make_contig(wl, "cpu", rotate=False)
    for r in range(host.n_rows):
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        host.pos[a:b] = torch.as_tensor(irregular_positions(b - a, r).astype(np.int32))
    cs, ms = oracle_centres(host)
    K = H.to_f64(host.K)
    pos = host.pos.numpy().astype(np.int64)
    got = gpu_score(to_dev(host), cs, ms, key_mode=PRE).cpu().numpy().astype(np.float64)
    for r in range(host.n_rows):
        li, s, h = host.row_lhs(r)
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        ref = oracle.row_scores(wl.theta, cs[li], ms[li], h, wl.group, K[a:b], pos[a:b], False,
                                int(host.p_now[s]), wl.offsets, "collapsed")
        bd = H.series_bound(wl.theta, cs[li], ms[li], h, wl.group, K[a:b], wl.offsets)
        assert H.score_error(got[a:b], ref, bd) <= 1e-4, r


# ------------------------------------------------------ GQA 8, 17 offsets

def test_group_of_eight_seventeen_offsets():
    wl = synth.WORKLOADS["qwen3_32b_128k"].with_(name="g8", n_layers=1, batch=2,
                                                  seq_len=(5000, 9000), n_calib=128)
    host = synth.make_contig(wl, "cpu")
    cs, ms = oracle_centres(host)
    rows = [0, 3, 9, 15]
    ref, bound = oracle_scores(host, cs, ms, tier="collapsed", rows=rows)
    got = gpu_score(to_dev(host), cs, ms).cpu().numpy().astype(np.float64)
    for r in rows:
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        assert H.score_error(got[a:b], ref[a:b], bound[a:b]) <= 1e-4


def test_zero_centre_heads():
    wl = synth.WORKLOADS["sweep_b64_adversarial"]
    z = wl.zero_centre_pairs()
    layer = int(np.nonzero(z.any(axis=1))[0][0])
    w = wl.with_(name=wl.name, batch=2, seq_len=(2000, 3000), n_calib=64)
    host = synth.make_contig(w, "cpu", layers=[layer])
    cs, ms = oracle_centres(host)
    ref, bound = oracle_scores(host, cs, ms, tier="collapsed")
    got = gpu_score(to_dev(host), cs, ms).cpu().numpy().astype(np.float64)
    assert H.score_error(got, ref, bound) <= 1e-4
    h = int(np.nonzero(z[layer])[0][0])
    a, b = host.row_off_np[h], host.row_off_np[h + 1]
    assert np.all(ref[a:b] >= 0)  # norm-only score of a zero-centre head


# --------------------------------------------------------------- paged

def paged_rows(p: synth.PagedCache, K_f64=None):
    """Host view of each (seq, head) row of a paged cache: (slots -> record index)."""
    bs = p.wl.block_size
    H_ = p.wl.n_kv_heads
    recs = []
    for s, n in enumerate(p.lens):
        j = np.arange(int(n))
        blk = p.block_table_np[s, j // bs].astype(np.int64)
        for h in range(H_):
            recs.append((blk * bs + j % bs) * H_ + h)
    return recs


@pytest.mark.parametrize("key_mode", [POST, PRE])
def test_paged_score_select_compact(key_mode):
    wl = synth.WORKLOADS["paged_16seq"].with_(name="paged_small", batch=5, seq_len=(40, 2100),
                                              n_calib=64)
    lens = np.array([40, 2100, 333, 1024, 1500])
    p = synth.make_paged(wl, "cpu", lens=lens)
    if key_mode == PRE:  # replace keys by pre-RoPE keys with the same positions
        contig = synth.make_contig(wl, "cpu", lens=lens, rotate=False, with_values=False)
        recs = paged_rows(p)
        K = p.K.view(-1, 128)
        for r, rec in enumerate(recs):
            a, b = contig.row_off_np[r], contig.row_off_np[r + 1]
            K[torch.as_tensor(rec)] = contig.K[a:b]
    qcal = synth.calib_queries(wl, 0, "cpu")[None]
    cs, ms = H.oracle_calibration(qcal)
    cs, ms = H.as_f32_exact(cs), H.as_f32_exact(ms)
    S, Hh = len(lens), wl.n_kv_heads
    row_off = synth.paged_row_offsets(lens, Hh)
    total = int(row_off[-1])
    Kf = H.to_f64(p.K).reshape(-1, 128)
    Kb = H.bits16(p.K).reshape(-1, 128)
    Vb = H.bits16(p.V).reshape(-1, 128)
    posf = p.pos.numpy().reshape(-1)
    recs = paged_rows(p)
    ref = np.empty(total)
    bound = np.empty(total)
    for r, rec in enumerate(recs):
        s, h = r // Hh, r % Hh
        a, b = row_off[r], row_off[r + 1]
        ref[a:b] = oracle.row_scores(wl.theta, cs[0], ms[0], h, wl.group, Kf[rec],
                                     posf[rec].astype(np.int64), key_mode == POST, int(lens[s]),
                                     wl.offsets, "literal")
        bound[a:b] = H.series_bound(wl.theta, cs[0], ms[0], h, wl.group, Kf[rec], wl.offsets)
    m = model_of(wl, 1)
    ro = torch.as_tensor(row_off, device=DEV)
    tbl = p.block_table.to(DEV)
    nb = p.K.shape[0]
    kv = tri.kv_paged(S, ro, total, tbl, wl.block_size, nb)
    Kd, Vd, pd = p.K.to(DEV), p.V.to(DEV), p.pos.to(DEV)
    B, W = 256, 32
    ws = tri.alloc_workspace(m, S, B)
    scores = torch.empty(total, dtype=torch.float32, device=DEV)
    tri.tri_score(m, kv, Kd, pd, torch.tensor(cs, dtype=torch.float32, device=DEV),
                  torch.tensor(ms, dtype=torch.float32, device=DEV), p.p_now.to(DEV), wl.offsets,
                  key_mode, scores, ws)
    got = scores.cpu().numpy().astype(np.float64)
    assert H.score_error(got, ref, bound) <= 1e-4
    # compaction into a fresh, shuffled block table, from the oracle's fp32 scores
    ref32 = H.as_f32_exact(ref)
    ob = (B + wl.block_size - 1) // wl.block_size
    n_out = S * ob + 3
    out_tbl = np.random.default_rng(9).permutation(n_out)[:S * ob].reshape(S, ob).astype(np.int32)
    otd = torch.as_tensor(out_tbl, device=DEV)
    Ko = torch.zeros(1, n_out, wl.block_size, Hh, 128, dtype=torch.bfloat16, device=DEV)
    Vo = torch.zeros_like(Ko)
    po = torch.full((1, n_out, wl.block_size, Hh), -1, dtype=torch.int32, device=DEV)
    kept = torch.full((S * Hh, B), -1, dtype=torch.int32, device=DEV)
    tri.tri_compact(m, kv, torch.tensor(ref32, dtype=torch.float32, device=DEV), B, W, Kd, Vd, pd,
                    tri.out_paged(otd, wl.block_size, n_out), Ko, Vo, po, kept, None, ws)
    st, flags = tri.tri_status_check(ws)
    assert st == 0, flags
    Kob = H.bits16(Ko).reshape(-1, 128)
    Vob = H.bits16(Vo).reshape(-1, 128)
    pob = po.cpu().numpy().reshape(-1)
    kept = kept.cpu().numpy()
    bs = wl.block_size
    for r, rec in enumerate(recs):
        s, h = r // Hh, r % Hh
        a, b = row_off[r], row_off[r + 1]
        sel = oracle.select(ref32[a:b], B, W)
        n = len(sel)
        np.testing.assert_array_equal(kept[r, :n], sel)
        i = np.arange(n)
        orec = (out_tbl[s, i // bs].astype(np.int64) * bs + i % bs) * Hh + h
        np.testing.assert_array_equal(Kob[orec], oracle.gather(Kb[rec], sel))
        np.testing.assert_array_equal(Vob[orec], oracle.gather(Vb[rec], sel))
        np.testing.assert_array_equal(pob[orec], oracle.gather(posf[rec], sel))


# ------------------------------------------------------------- flags

def test_device_flags_without_faults():
    """Bad block ids and inconsistent row offsets raise flags; nothing traps."""
    wl = synth.WORKLOADS["paged_16seq"].with_(name="flags", batch=2, seq_len=(64, 64), n_calib=16)
    lens = np.array([64, 64])
    p = synth.make_paged(wl, "cpu", lens=lens)
    S, Hh = 2, wl.n_kv_heads
    row_off = synth.paged_row_offsets(lens, Hh)
    total = int(row_off[-1])
    m = model_of(wl, 1)
    tbl = p.block_table.clone()
    tbl[1, 2] = 10 ** 6  # out of the pool
    kv = tri.kv_paged(S, torch.as_tensor(row_off, device=DEV), total, tbl.to(DEV), 16, p.K.shape[0])
    ws = tri.alloc_workspace(m, S, 32)
    c = torch.zeros(1, 32, 64, 2, device=DEV)
    n = torch.ones(1, 32, 64, device=DEV)
    scores = torch.empty(total, device=DEV)
    Kd = p.K.to(DEV)
    tri.tri_score(m, kv, Kd, None, c, n, p.p_now.to(DEV), wl.offsets, POST, scores, ws)
    st, flags = tri.tri_status_check(ws)
    assert flags & tri.TRI_FLAG_BLOCK_TABLE and st == 6
    st, flags = tri.tri_status_check(ws)  # cleared by the read
    assert st == 0 and flags == 0
    # total_keys inconsistent with row_off[R]
    kv2 = tri.kv_paged(S, torch.as_tensor(row_off, device=DEV), total - 5, p.block_table.to(DEV), 16,
                       p.K.shape[0])
    tri.tri_score(m, kv2, Kd, None, c, n, p.p_now.to(DEV), wl.offsets, POST, scores, ws)
    st, flags = tri.tri_status_check(ws)
    assert flags & tri.TRI_FLAG_ROW_OFFSETS
