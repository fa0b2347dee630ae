"""Decode attention over (compressed) caches against the oracle's softmax.

Tolerance from the arithmetic: each fp32 score s_j = scale * q.k_j carries an
error below eps_d = 4 d 2^-24 * scale * sum_i |q_i k_ji|; the output moves by at
most about 2 max_j eps_d * max|v| plus fp32 accumulation (1e-5 * max|v|), and
lse by max_j eps_d (+ 1e-6 relative)."""
import math

import numpy as np
import pytest
import torch

import kv_cache_compression_calib_b200 as tri
import oracle
import synth
from tests import harness as H
from tests.test_gpu_parity import model_of

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_attention(m, kv, K, V, q, scale, n_seqs, fn=None):
    L, S, Hq, d = q.shape
    out = torch.full((L, S, Hq, d), float("nan"), device=DEV)
    lse = torch.full((L, S, Hq), float("nan"), device=DEV)
    ws = tri.alloc_attention_workspace(m, n_seqs)
    (fn or tri.tri_decode_attention)(m, kv, K, V, q, scale, out, lse, ws)
    st, flags = tri.tri_status_check(ws)
    assert st == 0, flags
    return out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def check_row(out, lse, qf, keys, vals, scale, what):
    """out [d], lse: GPU result for one query; qf [d], keys/vals [n][d] float64 (generator bits)."""
    ref, rlse = oracle.attention(qf, keys, vals, scale)
    if len(keys) == 0:
        assert np.all(out == 0) and lse == -np.inf, what
        return
    d = len(qf)
    eps = 4 * d * 2.0 ** -24 * scale * np.max(np.abs(keys) @ np.abs(qf))
    vmax = np.max(np.abs(vals))
    assert np.max(np.abs(out - ref)) <= (2 * eps + 1e-5) * vmax + 1e-30, what
    assert abs(lse - rlse) <= eps + 1e-6 * abs(rlse) + 1e-6, what


@pytest.mark.parametrize("d,style,elem,hq", [(128, "half", "bf16", 32), (128, "half", "fp8", 32),
                                             (64, "interleaved", "bf16", 64), (256, "half", "bf16", 128),
                                             (256, "interleaved", "fp8", 16), (128, "half", "bf16", 8)])
def test_attention_contig(d, style, elem, hq):
    wl = synth.WORKLOADS["single_layer_4k"].with_(name=f"att{d}{style}{hq}", head_dim=d, rope_style=style,
                                                  n_q_heads=hq, batch=5, n_calib=8, theta=1e4 if d != 128 else 1e6)
    lens = [4096, 0, 1, 33, 700]
    host = synth.make_contig(wl, "cpu", lens=lens)
    if elem == "fp8":
        host.K, host.V = synth.to_fp8(host.K), synth.to_fp8(host.V)
    q = synth.decode_queries(wl, 0, np.asarray(lens), "cpu")[None]  # [1][S][Hq][d]
    scale = 1.0 / math.sqrt(d)
    m = model_of(wl, 1)
    kv = tri.kv_contig(len(lens), host.row_off.to(DEV), host.total, tri.elem_type_of(host.K))
    out, lse = run_attention(m, kv, host.K.to(DEV), host.V.to(DEV), q.to(DEV).contiguous(), scale, len(lens))
    K, V, qf = H.to_f64(host.K), H.to_f64(host.V), H.to_f64(q)
    G = wl.group
    for r in range(host.n_rows):
        _, s, h = host.row_lhs(r)
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        for g in range(G):
            qh = h * G + g
            check_row(out[0, s, qh], lse[0, s, qh], qf[0, s, qh], K[a:b], V[a:b], scale, (r, g))


@pytest.mark.parametrize("d,elem", [(128, "bf16"), (256, "bf16"), (64, "fp8"), (256, "fp8")])
def test_attention_paged(d, elem):
    """Paged caches (shuffled block table), ragged rows; head dim 256 runs the
    warp-pair form of the MMA kernel, fp8 its permuted-dim fragments."""
    wl = synth.WORKLOADS["paged_16seq"].with_(name=f"attp{d}{elem}", batch=3, n_calib=8, head_dim=d,
                                             theta=1e6 if d == 128 else 1e4)
    lens = np.array([300, 2100, 17])
    p = synth.make_paged(wl, "cpu", lens=lens)
    if elem == "fp8":
        p.K, p.V = synth.to_fp8(p.K), synth.to_fp8(p.V)
    S, Hh, bs = len(lens), wl.n_kv_heads, wl.block_size
    row_off = synth.paged_row_offsets(lens, Hh)
    m = model_of(wl, 1)
    kv = tri.kv_paged(S, torch.as_tensor(row_off, device=DEV), int(row_off[-1]), p.block_table.to(DEV), bs,
                      p.K.shape[0], tri.elem_type_of(p.K))
    q = synth.decode_queries(wl, 0, lens, "cpu")[None]
    scale = 1.0 / math.sqrt(d)
    out, lse = run_attention(m, kv, p.K.to(DEV), p.V.to(DEV), q.to(DEV).contiguous(), scale, S)
    Kf, Vf = H.to_f64(p.K).reshape(-1, d), H.to_f64(p.V).reshape(-1, d)
    qf = H.to_f64(q)
    G = wl.group
    for s in range(S):
        j = np.arange(int(lens[s]))
        blk = p.block_table_np[s, j // bs].astype(np.int64)
        for h in range(Hh):
            rec = (blk * bs + j % bs) * Hh + h
            for g in range(G):
                check_row(out[0, s, h * G + g], lse[0, s, h * G + g], qf[0, s, h * G + g], Kf[rec], Vf[rec], scale,
                          (s, h, g))


def test_attention_over_the_compacted_paged_cache():
    """Score -> compact into a fresh block table -> attend, against the oracle's
    selection, gather and softmax on the generator's bits (selection from the
    oracle's fp32 scores on both sides, as the compaction parity tests do)."""
    wl = synth.WORKLOADS["paged_16seq"].with_(name="attc", batch=3, n_calib=64)
    lens = np.array([5000, 2100, 700])
    p = synth.make_paged(wl, "cpu", lens=lens)
    qcal = synth.calib_queries(wl, 0, "cpu")[None]
    cs, ms = H.oracle_calibration(qcal)
    cs, ms = H.as_f32_exact(cs), H.as_f32_exact(ms)
    S, Hh, bs, d = len(lens), wl.n_kv_heads, wl.block_size, 128
    row_off = synth.paged_row_offsets(lens, Hh)
    total = int(row_off[-1])
    Kf, Vf = H.to_f64(p.K).reshape(-1, d), H.to_f64(p.V).reshape(-1, d)
    posf = p.pos.numpy().reshape(-1).astype(np.int64)
    recs, ref = [], np.empty(total)
    for s in range(S):
        j = np.arange(int(lens[s]))
        blk = p.block_table_np[s, j // bs].astype(np.int64)
        for h in range(Hh):
            rec = (blk * bs + j % bs) * Hh + h
            recs.append(rec)
            r = s * Hh + h
            ref[row_off[r]:row_off[r + 1]] = oracle.row_scores(wl.theta, cs[0], ms[0], h, wl.group, Kf[rec], posf[rec],
                                                               True, int(lens[s]), wl.offsets, "collapsed")
    ref32 = H.as_f32_exact(ref)
    m = model_of(wl, 1)
    kv = tri.kv_paged(S, torch.as_tensor(row_off, device=DEV), total, p.block_table.to(DEV), bs, p.K.shape[0])
    B, W = 1024, 128
    ws = tri.alloc_workspace(m, S, B)
    ob = B // bs
    n_out = S * ob
    out_tbl = np.random.default_rng(8).permutation(n_out).reshape(S, ob).astype(np.int32)
    Ko = torch.zeros(1, n_out, bs, Hh, d, dtype=torch.bfloat16, device=DEV)
    Vo = torch.zeros_like(Ko)
    tri.tri_compact(m, kv, torch.tensor(ref32, dtype=torch.float32, device=DEV), B, W, p.K.to(DEV), p.V.to(DEV),
                    None, tri.out_paged(torch.as_tensor(out_tbl, device=DEV), bs, n_out), Ko, Vo, None, None, None, ws)
    st, flags = tri.tri_status_check(ws)
    assert st == 0, flags
    # the compacted cache: every row of sequence s holds min(N_s, B) keys
    cnt = np.repeat(np.minimum(lens, B), Hh)
    row_off_c = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int64)
    kvc = tri.kv_paged(S, torch.as_tensor(row_off_c, device=DEV), int(row_off_c[-1]),
                       torch.as_tensor(out_tbl, device=DEV), bs, n_out)
    q = synth.decode_queries(wl, 0, lens, "cpu")[None]
    scale = 1.0 / math.sqrt(d)
    out, lse = run_attention(m, kvc, Ko, Vo, q.to(DEV).contiguous(), scale, S)
    qf = H.to_f64(q)
    G = wl.group
    for r, rec in enumerate(recs):
        s, h = r // Hh, r % Hh
        kept = oracle.select(ref32[row_off[r]:row_off[r + 1]], B, W)
        keys, vals = Kf[rec][kept], Vf[rec][kept]
        for g in range(G):
            check_row(out[0, s, h * G + g], lse[0, s, h * G + g], qf[0, s, h * G + g], keys, vals, scale, (r, g))


def test_attention_full_size_after_compaction():
    """The 36-layer 32K cache: score, compact to [R][2048], attend for all 1152 query
    heads in one call.  Sampled rows use the oracle's fp32 scores for the selection
    (so the kept set is the oracle's); the rest keep the GPU scores."""
    wl = synth.WORKLOADS["qwen3_8b_32k"]
    cache = synth.make_contig(wl, DEV)
    L, Hh, B, W, d = wl.n_layers, wl.n_kv_heads, wl.budget, wl.window, 128
    m = tri.model(L, wl.n_q_heads, Hh, wl.theta)
    kv = tri.kv_contig(1, cache.row_off, cache.total)
    c = torch.empty(L, wl.n_q_heads, 64, 2, device=DEV)
    n = torch.empty(L, wl.n_q_heads, 64, device=DEV)
    tri.tri_calib(m, cache.qcal, wl.n_calib, c, n)
    ws = tri.alloc_workspace(m, 1, B)
    scores = torch.empty(cache.total, device=DEV)
    tri.tri_score(m, kv, cache.K, cache.pos, c, n, cache.p_now, wl.offsets, tri.TRI_KEYS_POST_ROPE, scores, ws)
    rows = [3, 150]
    sampled = {}
    for r in rows:
        li, s, h = cache.row_lhs(r)
        a, b = cache.row_off_np[r], cache.row_off_np[r + 1]
        cs, ms = H.oracle_calibration(cache.qcal[li:li + 1])
        ref = H.as_f32_exact(oracle.row_scores(wl.theta, H.as_f32_exact(cs[0]), H.as_f32_exact(ms[0]), h, wl.group,
                                               H.to_f64(cache.K[a:b]), cache.pos[a:b].cpu().numpy().astype(np.int64),
                                               True, int(cache.lens[s]), wl.offsets, "collapsed"))
        scores[a:b] = torch.tensor(ref, dtype=torch.float32, device=DEV)
        sampled[r] = oracle.select(ref, B, W)
    R = cache.n_rows
    Ko = torch.empty(R, B, d, dtype=torch.bfloat16, device=DEV)
    Vo = torch.empty_like(Ko)
    tri.tri_compact(m, kv, scores, B, W, cache.K, cache.V, None, tri.out_contig(), Ko, Vo, None, None, None, ws)
    st, flags = tri.tri_status_check(ws)
    assert st == 0, flags
    kvc = tri.kv_contig(1, torch.arange(R + 1, device=DEV, dtype=torch.int64) * B, R * B)
    q = synth.decode_queries(wl, 0, np.asarray(cache.lens), DEV)  # layer 0's queries for every layer
    q = q[None].expand(L, -1, -1, -1).contiguous()
    scale = 1.0 / math.sqrt(d)
    out, lse = run_attention(m, kvc, Ko, Vo, q, scale, 1)
    qf = H.to_f64(q[0])
    G = wl.group
    for r in rows:
        li, s, h = cache.row_lhs(r)
        a = cache.row_off_np[r]
        keys = H.to_f64(cache.K[a + sampled[r]])
        vals = H.to_f64(cache.V[a + sampled[r]])
        for g in range(G):
            check_row(out[li, s, h * G + g], lse[li, s, h * G + g], qf[s, h * G + g], keys, vals, scale, (r, g))


@pytest.mark.parametrize("hq", [8, 32, 64, 128])
def test_attention_tensor_memory_kernel(hq):
    """tri_decode_attention_tc (tcgen05, bf16, head dim 128, contiguous): G = 1, 4, 8 and
    16 queries per KV head; rows empty, of one key, of exact multiples of the 128-key
    tile and with ragged tails, against the oracle."""
    wl = synth.WORKLOADS["single_layer_4k"].with_(name=f"atc{hq}", n_q_heads=hq, batch=7, n_calib=8)
    lens = [4096, 0, 1, 33, 700, 128, 256]
    host = synth.make_contig(wl, "cpu", lens=lens)
    q = synth.decode_queries(wl, 0, np.asarray(lens), "cpu")[None]
    scale = 1.0 / math.sqrt(128)
    m = model_of(wl, 1)
    kv = tri.kv_contig(len(lens), host.row_off.to(DEV), host.total)
    out, lse = run_attention(m, kv, host.K.to(DEV), host.V.to(DEV), q.to(DEV).contiguous(), scale, len(lens),
                             fn=tri.tri_decode_attention_tc)
    K, V, qf = H.to_f64(host.K), H.to_f64(host.V), H.to_f64(q)
    G = wl.group
    for r in range(host.n_rows):
        _, s_, h = host.row_lhs(r)
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        for g in range(G):
            qh = h * G + g
            check_row(out[0, s_, qh], lse[0, s_, qh], qf[0, s_, qh], K[a:b], V[a:b], scale, (r, g))


def test_attention_tensor_memory_kernel_refuses_other_caches():
    """Head dims other than 128, fp8 elements and paged caches are refused before any launch."""
    from kv_cache_compression_calib_b200 import _abi
    for d, elem in ((64, tri.TRI_ELEM_BF16), (128, tri.TRI_ELEM_FP8_E4M3)):
        m = tri.model(1, 32, 8, 1e6, head_dim=d)
        ro = torch.zeros(9, dtype=torch.int64, device=DEV)
        ro[1:] = 16
        kv = tri.kv_contig(1, ro, 16, elem)
        buf = torch.zeros(16 * d, dtype=torch.bfloat16, device=DEV)
        out = torch.zeros(32 * d, device=DEV)
        ws = tri.alloc_attention_workspace(m, 1)
        with pytest.raises(tri.TriError) as e:
            tri.tri_decode_attention_tc(m, kv, buf, buf, buf, 0.1, out, None, ws)
        assert e.value.status == _abi.TRI_ERR_UNSUPPORTED
