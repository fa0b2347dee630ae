"""Online centre update, concentration/drift statistics and pre-RoPE key centres
against the oracle.  Calibration statistics to 1e-6 of the mean norm (fp64 on
both sides, fp32 outputs); key centres to 2e-5 of the mean norm (fp32 Horner sums
along a lane's keys, settled with an exactly reduced phase every 8 batches and
at every irregular position step; fp64 sums across runs)."""
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


@pytest.mark.parametrize("decay,d,style", [(1.0, 128, "half"), (0.8, 128, "half"), (0.5, 64, "interleaved"),
                                           (0.95, 256, "half")])
def test_online_update_matches_weighted_oracle(decay, d, style):
    wl = synth.WORKLOADS["single_layer_4k"].with_(head_dim=d, rope_style=style, n_calib=160)
    q = synth.calib_queries(wl, 0, "cpu")[None]  # [1][Hq][160][d]
    sizes = [1, 64, 7, 88]
    m = model_of(wl, 1)
    Hq, F = wl.n_q_heads, d // 2
    sums = torch.zeros(1, Hq, F, 3, dtype=torch.float64, device=DEV)
    weight = torch.zeros(1, Hq, dtype=torch.float64, device=DEV)
    c = torch.empty(1, Hq, F, 2, device=DEV)
    n = torch.empty(1, Hq, F, device=DEV)
    off = 0
    for sz in sizes:
        tri.tri_calib_update(m, q[:, :, off:off + sz].to(DEV).contiguous(), sz, decay, sums, weight, c, n)
        off += sz
    c, n = c.cpu().numpy().astype(np.float64), n.cpu().numpy().astype(np.float64)
    qf = H.to_f64(q).reshape(1, Hq, 160, d)
    for g in range(Hq):
        batches, o = [], 0
        for sz in sizes:
            batches.append(qf[0, g, o:o + sz])
            o += sz
        rc, rm = oracle.calib_online(batches, decay, wl.interleaved)
        assert np.all(np.abs(c[0, g] - rc) <= 1e-6 * rm[:, None] + 1e-30), g
        assert np.all(np.abs(n[0, g] - rm) <= 1e-6 * rm), g
    w_ref = sum(sz * decay ** (len(sizes) - 1 - i) for i, sz in enumerate(sizes))
    np.testing.assert_allclose(weight.cpu().numpy(), w_ref, rtol=1e-15)


def test_calib_stats_match_oracle():
    wl = synth.WORKLOADS["sweep_b64_adversarial"]
    z = wl.zero_centre_pairs()
    layer = int(np.nonzero(z.any(axis=1))[0][0])  # a layer with zero-centre heads
    w = wl.with_(n_calib=256)
    cs, ms = H.oracle_calibration(synth.calib_queries(w, layer, "cpu")[None])
    rs, rms = H.oracle_calibration(synth.calib_queries(w.with_(seed=w.seed + 1), layer, "cpu")[None])
    cs, ms, rs, rms = (H.as_f32_exact(a) for a in (cs, ms, rs, rms))
    m = model_of(w, 1)
    Hq, F = w.n_q_heads, 64
    t = lambda a: torch.tensor(a, dtype=torch.float32, device=DEV)  # noqa: E731
    conc = torch.empty(1, Hq, F, device=DEV)
    hs = torch.empty(1, Hq, 2, device=DEV)
    tri.tri_calib_stats(m, Hq, t(cs), t(ms), t(rs), t(rms), conc, hs)
    conc, hs = conc.cpu().numpy(), hs.cpu().numpy()
    for g in range(Hq):
        rc, (rh, rd) = oracle.calib_stats(cs[0, g], ms[0, g], rs[0, g], rms[0, g])
        np.testing.assert_allclose(conc[0, g], rc, rtol=1e-6, atol=1e-7)
        np.testing.assert_allclose(hs[0, g], [rh, rd], rtol=1e-6, atol=1e-7)
    # without a reference: drift 0, concentration unchanged
    hs2 = torch.empty(1, Hq, 2, device=DEV)
    tri.tri_calib_stats(m, Hq, t(cs), t(ms), None, None, None, hs2)
    hs2 = hs2.cpu().numpy()
    assert np.all(hs2[..., 1] == 0) and np.array_equal(hs2[..., 0], hs[..., 0])
    # zero-centre query heads of this layer: their concentration is that of pure noise
    zq = np.repeat(z[layer], w.group)
    assert hs[0, zq, 0].max() < hs[0, ~zq, 0].min()


def run_key_centres(m, kv, K, pos, mode, R, F, n_seqs):
    c = torch.full((R, F, 2), float("nan"), device=DEV)
    n = torch.full((R, F), float("nan"), device=DEV)
    ws = tri.alloc_key_centres_workspace(m, n_seqs)
    tri.tri_key_centres(m, kv, K, pos, mode, c, n, ws)
    st, flags = tri.tri_status_check(ws)
    assert st == 0, flags
    return c.cpu().numpy().astype(np.float64), n.cpu().numpy().astype(np.float64)


def check_centres(c, n, rc, rm):
    scale = np.maximum(rm, 1e-30)
    assert np.all(np.abs(c - rc) <= 2e-5 * scale[:, None] + 1e-30)
    assert np.all(np.abs(n - rm) <= 2e-5 * scale + 1e-30)


@pytest.mark.parametrize("d,style,elem,mode", [(128, "half", "bf16", "post"), (128, "half", "bf16", "pre"),
                                               (64, "interleaved", "bf16", "post"),
                                               (256, "half", "fp8", "post"), (128, "interleaved", "fp8", "pre")])
def test_key_centres_contig(d, style, elem, mode):
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="kc", head_dim=d, rope_style=style, batch=3, n_calib=8,
                                                  theta=1e6 if d == 128 else 1e4)
    post = mode == "post"
    host = synth.make_contig(wl, "cpu", lens=[4096, 1000, 0], rotate=post)
    if elem == "fp8":
        host.K = synth.to_fp8(host.K)
    m = model_of(wl, 1)
    kv = tri.kv_contig(3, host.row_off.to(DEV), host.total, tri.elem_type_of(host.K))
    R, F = host.n_rows, d // 2
    kmode = tri.TRI_KEYS_POST_ROPE if post else tri.TRI_KEYS_PRE_ROPE
    Kd = host.K.to(DEV)
    # generator positions: the keys' own centres come back
    c0, _ = run_key_centres(m, kv, Kd, host.pos.to(DEV) if post else None, kmode, R, F, 3)
    # far positions (the same keys read as if cached at pos + 70000): the de-rotation
    # phase must be reduced exactly; compared against the oracle
    far = host.pos + 70000
    c, n = run_key_centres(m, kv, Kd, far.to(DEV) if post else None, kmode, R, F, 3)
    K = H.to_f64(host.K)
    pos = far.numpy().astype(np.int64)
    for r in range(R):
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        rc, rm = oracle.key_centres(wl.theta, K[a:b], pos[a:b], post, wl.interleaved)
        if b == a:
            assert np.all(c[r] == 0) and np.all(n[r] == 0)
        else:
            check_centres(c[r], n[r], rc, rm)
    # the generator's key centres (layer 0) are what the keys concentrate around
    heads = synth.layer_heads(wl, 0, "cpu")
    mu = np.stack([heads.key_re.numpy(), heads.key_im.numpy()], axis=-1)
    for h in range(wl.n_kv_heads):
        err = np.abs(c0[h] - mu[h]).max() / np.abs(mu[h]).max()
        assert err < 0.1, (h, err)



@pytest.mark.parametrize("elem,mode", [("bf16", "post"), ("fp8", "post"), ("bf16", "pre")])
def test_key_centres_short_rows_ragged_total(elem, mode):
    """One KV head, rows of 1001, 2, 37, 0 and 5 keys: chunks start at unaligned keys,
    rows shorter than a batch, and a total (1045) that is not a multiple of 4, so the
    last positions sit past the array's last whole 16-byte group."""
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="kc1", n_q_heads=4, n_kv_heads=1, batch=5, n_calib=8)
    post = mode == "post"
    lens = [1001, 2, 37, 0, 5]
    host = synth.make_contig(wl, "cpu", lens=lens, rotate=post)
    if elem == "fp8":
        host.K = synth.to_fp8(host.K)
    assert host.total == 1045
    m = model_of(wl, 1)
    kv = tri.kv_contig(len(lens), host.row_off.to(DEV), host.total, tri.elem_type_of(host.K))
    R, F = host.n_rows, 64
    kmode = tri.TRI_KEYS_POST_ROPE if post else tri.TRI_KEYS_PRE_ROPE
    far = host.pos + 123457
    c, n = run_key_centres(m, kv, host.K.to(DEV), far.to(DEV) if post else None, kmode, R, F, len(lens))
    K = H.to_f64(host.K)
    pos = far.numpy().astype(np.int64)
    for r in range(R):
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        if b == a:
            assert np.all(c[r] == 0) and np.all(n[r] == 0)
            continue
        rc, rm = oracle.key_centres(wl.theta, K[a:b], pos[a:b], post, wl.interleaved)
        check_centres(c[r], n[r], rc, rm)

def test_key_centres_irregular_positions():
    """RoPE caches with positions that break the regular stride (gaps, descending,
    repeated, across the int32 range's end): every such key settles the lane's
    Horner sum and restarts it."""
    from tests.test_gpu_parity import irregular_positions
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="kcirr", batch=1, n_calib=8)
    host = synth.make_contig(wl, "cpu", rotate=True)
    for r in range(host.n_rows):
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        host.pos[a:b] = torch.as_tensor(irregular_positions(b - a, r).astype(np.int32))
    m = model_of(wl, 1)
    kv = tri.kv_contig(1, host.row_off.to(DEV), host.total)
    c, n = run_key_centres(m, kv, host.K.to(DEV), host.pos.to(DEV), tri.TRI_KEYS_POST_ROPE, host.n_rows, 64, 1)
    K = H.to_f64(host.K)
    pos = host.pos.numpy().astype(np.int64)
    for r in range(host.n_rows):
        a, b = host.row_off_np[r], host.row_off_np[r + 1]
        rc, rm = oracle.key_centres(wl.theta, K[a:b], pos[a:b], True, wl.interleaved)
        check_centres(c[r], n[r], rc, rm)


def test_key_centres_paged():
    wl = synth.WORKLOADS["paged_16seq"].with_(name="kcp", batch=3, n_calib=8)
    lens = np.array([300, 2100, 1024])
    p = synth.make_paged(wl, "cpu", lens=lens)
    S, Hh, bs = len(lens), wl.n_kv_heads, wl.block_size
    row_off = synth.paged_row_offsets(lens, Hh)
    m = model_of(wl, 1)
    kv = tri.kv_paged(S, torch.as_tensor(row_off, device=DEV), int(row_off[-1]), p.block_table.to(DEV), bs,
                      p.K.shape[0])
    c, n = run_key_centres(m, kv, p.K.to(DEV), p.pos.to(DEV), tri.TRI_KEYS_POST_ROPE, S * Hh, 64, S)
    Kf = H.to_f64(p.K).reshape(-1, 128)
    posf = p.pos.numpy().reshape(-1).astype(np.int64)
    for s in range(S):
        j = np.arange(int(lens[s]))
        blk = p.block_table_np[s, j // bs].astype(np.int64)
        for h in range(Hh):
            rec = (blk * bs + j % bs) * Hh + h
            rc, rm = oracle.key_centres(wl.theta, Kf[rec], posf[rec], True)
            check_centres(c[s * Hh + h], n[s * Hh + h], rc, rm)


def test_key_centres_full_size_sampled():
    """All 288 rows of the 36-layer 32K cache in one call; rows sampled against the oracle."""
    wl = synth.WORKLOADS["qwen3_8b_32k"]
    cache = synth.make_contig(wl, DEV, with_values=False)
    m = tri.model(wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.theta)
    kv = tri.kv_contig(1, cache.row_off, cache.total)
    c, n = run_key_centres(m, kv, cache.K, cache.pos, tri.TRI_KEYS_POST_ROPE, cache.n_rows, 64, 1)
    for r in (0, 101, 287):
        a, b = cache.row_off_np[r], cache.row_off_np[r + 1]
        rc, rm = oracle.key_centres(wl.theta, H.to_f64(cache.K[a:b]), cache.pos[a:b].cpu().numpy().astype(np.int64),
                                    True)
        check_centres(c[r], n[r], rc, rm)
