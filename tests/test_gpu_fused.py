"""tri_score_compact: scoring and selection fused on chip (rows up to 32768 keys).

The fused kernel runs the score kernel's arithmetic in the same reduction
order, so its scores, kept sets and compacted caches must equal tri_score +
tri_compact bit for bit; against the oracle the scores meet the score
tolerance and the kept sets the tie rule, as for the unfused path."""
import numpy as np
import pytest
import torch

import kv_cache_compression_calib_b200 as tri
import synth
from tests import harness as H
from tests.test_gpu_parity import POST, PRE, model_of, oracle_centres, oracle_scores

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_both(wl, cache, cs, ms, B, W, key_mode=POST, out_paged=None, max_row_len=None, fused_scores=True):
    """(fused, unfused) results on a contiguous device cache.  fused_scores=False
    passes no score buffer to tri_score_compact (the fused kernel for any row up to
    TRI_FUSED_MAX_ROW keys; its scores are then compared through the kept sets)."""
    m = model_of(wl, len(cache.layers))
    S, R, d = len(cache.lens), cache.n_rows, wl.head_dim
    kv = tri.kv_contig(S, cache.row_off, cache.total, tri.elem_type_of(cache.K))
    c32 = torch.tensor(cs, dtype=torch.float32, device=DEV)
    m32 = torch.tensor(ms, dtype=torch.float32, device=DEV)
    res = []
    for fused in (True, False):
        ws = tri.alloc_workspace(m, S, B)
        scores = torch.full((max(cache.total, 1),), float("nan"), device=DEV)
        Ko = torch.zeros(R, B, d, dtype=cache.K.dtype, device=DEV)
        Vo = torch.zeros_like(Ko)
        po = torch.full((R, B), -7, dtype=torch.int32, device=DEV)
        kept = torch.full((R, B), -1, dtype=torch.int32, device=DEV)
        cnt = torch.full((R,), -1, dtype=torch.int32, device=DEV)
        if fused:
            mrl = int(np.diff(cache.row_off_np).max()) if max_row_len is None else max_row_len
            tri.tri_score_compact(m, kv, cache.K, cache.V, cache.pos, c32, m32, cache.p_now, wl.offsets, key_mode, B,
                                  W, mrl, tri.out_contig(), Ko, Vo, po, kept, cnt, scores if fused_scores else None,
                                  ws)
        else:
            tri.tri_score(m, kv, cache.K, cache.pos, c32, m32, cache.p_now, wl.offsets, key_mode, scores, ws)
            tri.tri_compact(m, kv, scores, B, W, cache.K, cache.V, cache.pos, tri.out_contig(), Ko, Vo, po, kept,
                            cnt, ws)
        st, flags = tri.tri_status_check(ws)
        res.append(dict(st=st, flags=flags, scores=scores.cpu(), K=Ko.cpu(), V=Vo.cpu(), pos=po.cpu(),
                        kept=kept.cpu().numpy(), cnt=cnt.cpu().numpy()))
    return res


def assert_identical(a, b, scores=True):
    assert a["st"] == b["st"] == 0, (a["flags"], b["flags"])
    if scores:
        assert torch.equal(a["scores"].view(torch.int32), b["scores"].view(torch.int32))
    np.testing.assert_array_equal(a["kept"], b["kept"])
    np.testing.assert_array_equal(a["cnt"], b["cnt"])
    assert torch.equal(H.torch_bits(a["K"]), H.torch_bits(b["K"]))
    assert torch.equal(H.torch_bits(a["V"]), H.torch_bits(b["V"]))
    assert torch.equal(a["pos"], b["pos"])


@pytest.mark.parametrize("d,style,elem,mode", [(128, "half", "bf16", POST), (128, "half", "bf16", PRE),
                                               (128, "half", "fp8", POST), (64, "interleaved", "bf16", POST),
                                               (256, "half", "bf16", POST), (256, "interleaved", "fp8", PRE),
                                               (64, "half", "bf16", PRE), (64, "interleaved", "fp8", POST),
                                               (256, "half", "bf16", PRE)])
def test_fused_equals_two_calls_and_meets_the_oracle(d, style, elem, mode):
    wl = synth.WORKLOADS["single_layer_4k"].with_(name=f"fz{d}{style}", head_dim=d, rope_style=style, batch=6,
                                                  n_calib=64, theta=1e6 if d == 128 else 1e4)
    lens = [4096, 1000, 37, 512, 513, 0]
    host = synth.make_contig(wl, "cpu", lens=lens, rotate=(mode == POST))
    if elem == "fp8":
        host.K, host.V = synth.to_fp8(host.K), synth.to_fp8(host.V)
    cs, ms = oracle_centres(host)
    from tests.test_gpu_parity import to_dev
    dev = to_dev(host)
    B, W = 512, 64
    fused, plain = run_both(wl, dev, cs, ms, B, W, key_mode=mode)
    assert_identical(fused, plain)
    # against the oracle: scores, and kept sets within the tie rule
    ref, bound = oracle_scores(host, cs, ms, post_rope=(mode == POST), tier="collapsed")
    got = fused["scores"].numpy().astype(np.float64)[:host.total]
    assert H.score_error(got, ref, bound) <= 1e-4
    Kb = H.raw_bits(host.K)
    for r in range(host.n_rows):
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        n = min(b - a, B)
        H.check_kept_within_ties(fused["kept"][r, :n], ref[a:b], B, W, bound[a:b])
        np.testing.assert_array_equal(H.raw_bits(fused["K"][r, :n]), Kb[a:b][fused["kept"][r, :n]])


def test_fused_special_rows():
    """B == W (window only), W == 0, N == B, N == B + 1, constant and tied scores."""
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="fzs", batch=4, n_calib=16)
    host = synth.make_contig(wl, "cpu", lens=[300, 257, 256, 2000])
    # ties: duplicate whole keys so many scores are exactly equal
    K = host.K.view(-1, 128)
    K[host.row_off_np[8]:host.row_off_np[9]] = K[host.row_off_np[8]]
    from tests.test_gpu_parity import to_dev
    cs, ms = oracle_centres(host)
    dev = to_dev(host)
    for B, W in ((256, 256), (256, 0), (256, 31), (1, 1), (1, 0)):
        fused, plain = run_both(wl, dev, cs, ms, B, W)
        assert_identical(fused, plain)


def test_fused_fallback_and_long_rows():
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="fzl", batch=2, n_calib=16)
    host = synth.make_contig(wl, "cpu", lens=[40000, 3000])
    from tests.test_gpu_parity import to_dev
    cs, ms = oracle_centres(host)
    dev = to_dev(host)
    fused, plain = run_both(wl, dev, cs, ms, 2048, 128)  # max_row_len 40000: the two-call path
    assert_identical(fused, plain)
    # a bound below the real row length: the long rows are flagged, the rest done
    m = model_of(wl, 1)
    kv = tri.kv_contig(2, dev.row_off, dev.total)
    ws = tri.alloc_workspace(m, 2, 2048)
    Ko = torch.zeros(dev.n_rows, 2048, 128, dtype=torch.bfloat16, device=DEV)
    Vo = torch.zeros_like(Ko)
    cnt = torch.full((dev.n_rows,), -1, dtype=torch.int32, device=DEV)
    kept = torch.full((dev.n_rows, 2048), 12345, dtype=torch.int32, device=DEV)
    tri.tri_score_compact(m, kv, dev.K, dev.V, None, torch.tensor(cs, dtype=torch.float32, device=DEV),
                          torch.tensor(ms, dtype=torch.float32, device=DEV), dev.p_now, wl.offsets, POST, 2048, 128,
                          32768, tri.out_contig(), Ko, Vo, None, kept, cnt, None, ws)
    st, flags = tri.tri_status_check(ws)
    assert st == tri._abi.TRI_ERR_DEVICE_FLAG and flags == tri.TRI_FLAG_ROW_OFFSETS
    c = cnt.cpu().numpy()
    assert np.all(c[:8] == 0) and np.all(c[8:] == 2048)
    # the flagged rows keep nothing: kept entries emptied, output records untouched
    assert np.all(kept[:8].cpu().numpy() == -1)
    assert not Ko[:8].any() and not Vo[:8].any()
    np.testing.assert_array_equal(H.raw_bits(Ko[8:].cpu()), plain_rows(plain, 8))
    np.testing.assert_array_equal(kept[8:].cpu().numpy(), plain["kept"][8:])


@pytest.mark.parametrize("d,elem", [(128, "bf16"), (256, "bf16"), (128, "fp8")])
def test_fused_rows_beyond_the_stated_bound(d, elem):
    """max_row_len 4096 against rows of 100 to 32768 keys: the call takes the fused
    kernel and every row up to TRI_FUSED_MAX_ROW is processed normally, equal to
    tri_score + tri_compact bit for bit."""
    wl = synth.WORKLOADS["single_layer_4k"].with_(name=f"fzbound{d}{elem}", head_dim=d, batch=6, n_calib=16,
                                                  theta=1e6 if d == 128 else 1e4)
    host = synth.make_contig(wl, "cpu", lens=[20480, 20481, 24000, 32768, 2176, 100])
    if elem == "fp8":
        host.K, host.V = synth.to_fp8(host.K), synth.to_fp8(host.V)
    from tests.test_gpu_parity import to_dev
    cs, ms = oracle_centres(host)
    dev = to_dev(host)
    fused, plain = run_both(wl, dev, cs, ms, 2048, 128, max_row_len=4096)
    assert_identical(fused, plain)


def paged_both(wl, lens, B, W, elem="bf16", edit_table=None):
    """(fused, unfused) results of one paged re-score round (post-RoPE keys,
    contiguous [R][B] outputs): (status, flags, scores, kept, K, V, pos) each, and
    the row offsets."""
    p = synth.make_paged(wl, "cpu", lens=lens)
    if elem == "fp8":
        p.K, p.V = synth.to_fp8(p.K), synth.to_fp8(p.V)
    qcal = synth.calib_queries(wl, 0, "cpu")[None]
    cs, ms = H.oracle_calibration(qcal)
    cs, ms = H.as_f32_exact(cs), H.as_f32_exact(ms)
    S, Hh, bs, d = len(lens), wl.n_kv_heads, wl.block_size, wl.head_dim
    row_off = synth.paged_row_offsets(np.asarray(lens), Hh)
    total = int(row_off[-1])
    m = model_of(wl, 1)
    tbl = p.block_table.clone()
    if edit_table:
        edit_table(tbl)
    kv = tri.kv_paged(S, torch.as_tensor(row_off, device=DEV), total, tbl.to(DEV), bs, p.K.shape[0],
                      tri.elem_type_of(p.K))
    Kd, Vd, pd = p.K.to(DEV), p.V.to(DEV), p.pos.to(DEV)
    c32 = torch.tensor(cs, dtype=torch.float32, device=DEV)
    m32 = torch.tensor(ms, dtype=torch.float32, device=DEV)
    res = []
    for fused in (True, False):
        ws = tri.alloc_workspace(m, S, B)
        scores = torch.full((total,), float("nan"), device=DEV)
        Ko = torch.zeros(S * Hh, B, d, dtype=Kd.dtype, device=DEV)
        Vo = torch.zeros_like(Ko)
        po = torch.full((S * Hh, B), -1, dtype=torch.int32, device=DEV)
        kept = torch.full((S * Hh, B), -1, dtype=torch.int32, device=DEV)
        if fused:
            tri.tri_score_compact(m, kv, Kd, Vd, pd, c32, m32, p.p_now.to(DEV), wl.offsets, POST, B, W,
                                  int(max(lens)), tri.out_contig(), Ko, Vo, po, kept, None, scores, ws)
        else:
            tri.tri_score(m, kv, Kd, pd, c32, m32, p.p_now.to(DEV), wl.offsets, POST, scores, ws)
            tri.tri_compact(m, kv, scores, B, W, Kd, Vd, pd, tri.out_contig(), Ko, Vo, po, kept, None, ws)
        st, flags = tri.tri_status_check(ws)
        res.append((st, flags, scores.cpu(), kept.cpu(), H.torch_bits(Ko.cpu()), H.torch_bits(Vo.cpu()), po.cpu()))
    return res, row_off


def assert_same_round(a, b):
    for x, y in zip(a, b):
        if isinstance(x, torch.Tensor):
            assert torch.equal(x.view(torch.int32) if x.dtype == torch.float32 else x,
                               y.view(torch.int32) if y.dtype == torch.float32 else y)
        else:
            assert x == y


@pytest.mark.parametrize("d,style,elem", [(128, "half", "bf16"), (64, "interleaved", "bf16"), (256, "half", "bf16"),
                                          (128, "half", "fp8"), (128, "interleaved", "fp8"), (256, "interleaved", "bf16")])
def test_fused_paged_rounds_equal_two_calls(d, style, elem):
    """Paged re-score rounds (rows of a few thousand keys: several batches per warp,
    partial batches at the row ends) at every head dim, pairing and element type:
    fused equals tri_score + tri_compact bit for bit."""
    wl = synth.WORKLOADS["paged_16seq"].with_(name=f"fzpr{d}{style}{elem}", batch=3, n_calib=16, head_dim=d,
                                              rope_style=style, theta=1e6 if d == 128 else 1e4)
    (f, u), _ = paged_both(wl, [2176, 3000, 700], 2048, 128, elem)
    assert f[0] == u[0] == 0, (f[1], u[1])
    assert_same_round(f, u)


def test_fused_paged_unplaceable_block():
    """Block ids outside the pool inside whole batches: the fused kernel scores
    those keys 0 and raises the same flag as the score kernel; results equal
    tri_score + tri_compact."""
    wl = synth.WORKLOADS["paged_16seq"].with_(name="fzpb", batch=2, n_calib=16)
    bs = wl.block_size

    def edit(tbl):
        tbl[0, 5] = 10 ** 6  # keys 80 .. 95 of sequence 0: out of the pool
        tbl[1, 63] = -3      # the last block of sequence 1

    (f, u), row_off = paged_both(wl, [2176, 1024], 1024, 64, edit_table=edit)
    assert f[1] == u[1] == tri.TRI_FLAG_BLOCK_TABLE and f[0] == u[0] == tri._abi.TRI_ERR_DEVICE_FLAG
    bad = np.zeros(int(row_off[-1]), dtype=bool)
    for s, blk in ((0, 5), (1, 63)):
        for h in range(wl.n_kv_heads):
            r0 = int(row_off[s * wl.n_kv_heads + h])
            bad[r0 + blk * bs: r0 + (blk + 1) * bs] = True
    assert torch.all(f[2][torch.as_tensor(bad)] == 0)  # unplaceable keys score 0 on both paths
    assert_same_round(f, u)


def plain_rows(res, r0):
    return H.raw_bits(res["K"][r0:])


def test_fused_paged():
    wl = synth.WORKLOADS["paged_16seq"].with_(name="fzp", batch=3, n_calib=32)
    lens = np.array([300, 2100, 1024])
    p = synth.make_paged(wl, "cpu", lens=lens)
    qcal = synth.calib_queries(wl, 0, "cpu")[None]
    cs, ms = H.oracle_calibration(qcal)
    cs, ms = H.as_f32_exact(cs), H.as_f32_exact(ms)
    S, Hh, bs = len(lens), wl.n_kv_heads, wl.block_size
    row_off = synth.paged_row_offsets(lens, Hh)
    total = int(row_off[-1])
    m = model_of(wl, 1)
    kv = tri.kv_paged(S, torch.as_tensor(row_off, device=DEV), total, p.block_table.to(DEV), bs, p.K.shape[0])
    Kd, Vd, pd = p.K.to(DEV), p.V.to(DEV), p.pos.to(DEV)
    B, W = 256, 32
    ob = B // bs
    n_out = S * ob
    out_tbl = torch.as_tensor(np.random.default_rng(4).permutation(n_out).reshape(S, ob).astype(np.int32),
                              device=DEV)
    res = []
    for fused in (True, False):
        ws = tri.alloc_workspace(m, S, B)
        scores = torch.empty(total, device=DEV)
        Ko = torch.zeros(1, n_out, bs, Hh, 128, dtype=torch.bfloat16, device=DEV)
        Vo = torch.zeros_like(Ko)
        po = torch.full((1, n_out, bs, Hh), -1, dtype=torch.int32, device=DEV)
        kept = torch.full((S * Hh, B), -1, dtype=torch.int32, device=DEV)
        c32 = torch.tensor(cs, dtype=torch.float32, device=DEV)
        m32 = torch.tensor(ms, dtype=torch.float32, device=DEV)
        if fused:
            tri.tri_score_compact(m, kv, Kd, Vd, pd, c32, m32, p.p_now.to(DEV), wl.offsets, POST, B, W,
                                  int(lens.max()), tri.out_paged(out_tbl, bs, n_out), Ko, Vo, po, kept, None, scores,
                                  ws)
        else:
            tri.tri_score(m, kv, Kd, pd, c32, m32, p.p_now.to(DEV), wl.offsets, POST, scores, ws)
            tri.tri_compact(m, kv, scores, B, W, Kd, Vd, pd, tri.out_paged(out_tbl, bs, n_out), Ko, Vo, po, kept,
                            None, ws)
        st, flags = tri.tri_status_check(ws)
        assert st == 0, flags
        res.append((scores.cpu(), kept.cpu(), H.torch_bits(Ko.cpu()), H.torch_bits(Vo.cpu()), po.cpu()))
    for a, b in zip(*res):
        assert torch.equal(a.view(torch.int32) if a.dtype == torch.float32 else a,
                           b.view(torch.int32) if b.dtype == torch.float32 else b)


def test_fused_full_size_equals_two_calls():
    """The 36-layer 32K cache in one fused call (288 rows of 32768 keys, scores kept
    on chip) against tri_score + tri_compact, and sampled rows against the oracle."""
    wl = synth.WORKLOADS["qwen3_8b_32k"]
    cache = synth.make_contig(wl, DEV)
    L = wl.n_layers
    m = tri.model(L, wl.n_q_heads, wl.n_kv_heads, wl.theta)
    c = torch.empty(L, wl.n_q_heads, 64, 2, device=DEV)
    n = torch.empty(L, wl.n_q_heads, 64, device=DEV)
    tri.tri_calib(m, cache.qcal, wl.n_calib, c, n)
    cs, ms = c.cpu().numpy().astype(np.float64), n.cpu().numpy().astype(np.float64)  # both paths use these
    B, W = wl.budget, wl.window
    fused, plain = run_both(wl, cache, cs, ms, B, W, fused_scores=False)  # 32768-key rows: the fused kernel
    assert_identical(fused, plain, scores=False)
    for r in (0, 211):
        li, s, h = cache.row_lhs(r)
        a, b = cache.row_off_np[r], cache.row_off_np[r + 1]
        ocs, oms = H.oracle_calibration(cache.qcal[li:li + 1])
        ocs, oms = H.as_f32_exact(ocs[0]), H.as_f32_exact(oms[0])
        Kf = H.to_f64(cache.K[a:b])
        ref = oracle_row(wl, ocs, oms, h, Kf, cache, a, b, s)
        bd = H.series_bound(wl.theta, ocs, oms, h, wl.group, Kf, wl.offsets)
        H.check_kept_within_ties(fused["kept"][r], ref, B, W, bd)


def oracle_row(wl, cs, ms, h, Kf, cache, a, b, s):
    import oracle
    return oracle.row_scores(wl.theta, cs, ms, h, wl.group, Kf, cache.pos[a:b].cpu().numpy().astype(np.int64), True,
                             int(cache.lens[s]), wl.offsets, "collapsed")
