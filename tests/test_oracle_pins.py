"""Pins of the CPU oracle against things other than itself.

Every check here is independent of the oracle's own formulas:
  * explicit RoPE rotations and dot products (numpy, long double) - the
    closed form the trig series must equal at every token distance;
  * hand-worked closed forms (tests/golden/closed_forms.json);
  * special cases that reduce the score to a textbook attention-logit sum or
    to a pure norm sum;
  * numpy's mean / lexsort / fancy indexing as second implementations of the
    calibration, selection and gather;
  * brute force on tiny rows, and invariants that must hold at any size.

Sources: "TriAttention：基于三角函数 KV 压缩的高效长推理" (whatsmy.fun paper
digest), section 流程详解 steps 1-4; "WeianMao/triattention" project card,
"How it works".
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

LD = np.longdouble
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


# ----------------------------------------------------------- explicit RoPE

def omega_ld(theta, d):
    f = np.arange(d // 2, dtype=LD)
    return np.power(LD(theta), -LD(2) * f / LD(d))


def rope_ld(x, p, theta):
    """Rotate-half RoPE of vector(s) x [..., d] at position p, in long double.

    x'[f] = x[f] cos(w_f p) - x[f+F] sin(w_f p);  x'[f+F] = x[f+F] cos + x[f] sin."""
    x = np.asarray(x, dtype=LD)
    d = x.shape[-1]
    F = d // 2
    a = omega_ld(theta, d) * LD(p)
    c, s = np.cos(a), np.sin(a)
    out = np.empty_like(x)
    out[..., :F] = x[..., :F] * c - x[..., F:] * s
    out[..., F:] = x[..., F:] * c + x[..., :F] * s
    return out


def rope_il_ld(x, p, theta):
    """Interleaved RoPE (GPT-J / Meta-Llama complex layout) of x [..., d] at position p:
    x'[2f] = x[2f] cos(w_f p) - x[2f+1] sin(w_f p);  x'[2f+1] = x[2f+1] cos + x[2f] sin."""
    x = np.asarray(x, dtype=LD)
    d = x.shape[-1]
    a = omega_ld(theta, d) * LD(p)
    c, s = np.cos(a), np.sin(a)
    out = np.empty_like(x)
    out[..., 0::2] = x[..., 0::2] * c - x[..., 1::2] * s
    out[..., 1::2] = x[..., 1::2] * c + x[..., 0::2] * s
    return out


def pair_abs_il(x):
    x = np.asarray(x, dtype=np.float64)
    return np.hypot(x[..., 0::2], x[..., 1::2])


def as_centre_il(v):
    v = np.asarray(v, dtype=np.float64)
    return np.stack([v[..., 0::2], v[..., 1::2]], axis=-1)


def dot_ld(a, b):
    return np.sum(np.asarray(a, dtype=LD) * np.asarray(b, dtype=LD), axis=-1)


def pair_abs(x):
    x = np.asarray(x, dtype=np.float64)
    F = x.shape[-1] // 2
    return np.hypot(x[..., :F], x[..., F:])


def as_centre(v):
    """Vector [d] -> centre [F][2] (pair f = dims (f, f+F))."""
    v = np.asarray(v, dtype=np.float64)
    F = v.shape[-1] // 2
    return np.stack([v[..., :F], v[..., F:]], axis=-1)


# ------------------------------------------------------------------- omega

def test_omega_is_theta_power():
    d, theta = 128, 1e6
    w = oracle.omega(theta, d)
    assert w[0] == 1.0
    # w_32 = theta^(-64/128) = theta^(-1/2) = 1e-3: catches an exponent of -f/d
    assert abs(w[32] - 1e-3) < 1e-18
    f = np.arange(d // 2)
    np.testing.assert_allclose(np.log(w) / np.log(theta), -2 * f / d, rtol=0, atol=1e-15)


# ------------------------------------------- trig series == RoPE logit (1e-12)

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_trig_series_equals_rope_dot_at_every_distance(seed):
    """sum_f |q_f||k_f| cos(w_f (p-j) + arg q_f - arg k_f) == RoPE(q,p) . RoPE(k,j).

    Distances cover 0..4100 densely and a sweep up to 2^17 + 2^16, through
    several (p, j) pairs per distance, to 1e-12 of sum_f |q_f||k_f|."""
    rng = np.random.default_rng(seed)
    d, theta = 128, 1e6
    q = rng.standard_normal(d) * np.exp(rng.standard_normal(d))
    k = rng.standard_normal(d) * np.exp(rng.standard_normal(d))
    scale = float(np.sum(pair_abs(q) * pair_abs(k)))
    qb = as_centre(q)
    dists = list(range(0, 4101, 7)) + list(rng.integers(0, 2**17 + 2**16, size=60))
    worst = 0.0
    for dist in dists:
        dist = int(dist)
        for j in (0, 12345, 131071 - min(dist, 131071) // 2):
            p = j + dist
            ref = dot_ld(rope_ld(q, p, theta), rope_ld(k, j, theta))
            got = oracle.trig_series(theta, qb, k, dist)
            worst = max(worst, abs(float(ref) - got) / scale)
    assert worst < 1e-12, worst


@pytest.mark.parametrize("d,interleaved", [(64, False), (256, False), (64, True), (128, True),
                                           (256, True)])
def test_trig_series_equals_rope_dot_other_layouts(d, interleaved):
    """The same identity for head dims 64 and 256 and for interleaved pairs (2f, 2f+1),
    against an explicit rotation of the matching layout."""
    rng = np.random.default_rng(d + 7 * interleaved)
    theta = 1e4 if d == 256 else 1e6
    rope = rope_il_ld if interleaved else rope_ld
    pabs = pair_abs_il if interleaved else pair_abs
    q = rng.standard_normal(d) * np.exp(rng.standard_normal(d))
    k = rng.standard_normal(d) * np.exp(rng.standard_normal(d))
    scale = float(np.sum(pabs(q) * pabs(k)))
    qb = as_centre_il(q) if interleaved else as_centre(q)
    worst = 0.0
    for dist in list(range(0, 600, 13)) + list(rng.integers(0, 2**17, size=20)):
        dist = int(dist)
        for j in (0, 4099):
            ref = dot_ld(rope(q, j + dist, theta), rope(k, j, theta))
            got = oracle.trig_series(theta, qb, k, dist, interleaved=interleaved)
            worst = max(worst, abs(float(ref) - got) / scale)
    assert worst < 1e-12, worst


def test_trig_series_negative_distance():
    rng = np.random.default_rng(7)
    d, theta = 128, 1e6
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    scale = float(np.sum(pair_abs(q) * pair_abs(k)))
    for dist in (-1, -17, -4096, -100000):
        ref = dot_ld(rope_ld(q, 200000 + dist, theta), rope_ld(k, 200000, theta))
        got = oracle.trig_series(theta, as_centre(q), k, dist)
        assert abs(float(ref) - got) / scale < 1e-12


# ------------------------------------------------------- hand-worked goldens

def test_golden_closed_forms():
    with open(GOLDEN) as fh:
        cases = json.load(fh)["cases"]
    assert len(cases) >= 5
    for c in cases:
        qb = np.array(c["qbar"], dtype=np.float64)
        mn = np.array(c["mnorm"], dtype=np.float64)
        keys = np.array(c["keys"], dtype=np.float64)
        expect = np.array([eval(e, {"math": math}) for e in c["expect"]])
        for fn in (oracle.score_literal, oracle.score_collapsed, oracle.score_absorbed):
            got = fn(c["theta"], qb, mn, keys, c["pos"], False, c["p_now"], c["offsets"])
            np.testing.assert_allclose(got, expect, rtol=1e-14, atol=1e-14, err_msg=c["name"])


# ------------------------------------- whole score: textbook special cases

def _explicit_logit_sum(qs, k_cached, pos, post_rope, p_now, offsets, theta, rope=rope_ld):
    """(1/G) sum_g sum_delta RoPE(q_g, p_now+delta) . k_post, k_post = the key as RoPE'd at pos."""
    k_post = np.asarray(k_cached, dtype=LD) if post_rope else rope(k_cached, pos, theta)
    tot = LD(0)
    for q in qs:
        for dlt in offsets:
            tot += dot_ld(rope(q, p_now + dlt, theta), k_post)
    return tot / LD(len(qs))


@pytest.mark.parametrize("post_rope", [True, False])
def test_identical_queries_give_attention_logit_sum(post_rope):
    """All calibration queries of a head identical => E|q_f| = |qbar_f|, the norm term
    vanishes and the score is the textbook sum of RoPE attention logits over the
    future positions p_now + delta, averaged over the G query heads."""
    rng = np.random.default_rng(11)
    d, theta, G, nq = 128, 1e6, 3, 5
    offsets = [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096]
    qs = rng.standard_normal((G, d))
    centres, mnorms = [], []
    for g in range(G):
        c, m = oracle.calib(np.repeat(qs[g][None], nq, axis=0))
        centres.append(c)
        mnorms.append(m)
    centres, mnorms = np.array(centres), np.array(mnorms)
    n = 24
    pos = rng.integers(0, 40000, size=n)
    p_now = 40000
    keys_pre = rng.standard_normal((n, d)) * 0.5
    keys = np.array([rope_ld(keys_pre[j], pos[j], theta) for j in range(n)], dtype=np.float64) \
        if post_rope else keys_pre
    ref = np.array([float(_explicit_logit_sum(qs, keys[j], pos[j], post_rope, p_now, offsets,
                                              theta)) for j in range(n)])
    scale = np.array([len(offsets) * np.mean([np.sum(pair_abs(q) * pair_abs(keys[j])) for q in qs])
                      for j in range(n)])
    for tier in ("literal", "collapsed", "absorbed"):
        fn = getattr(oracle, "score_" + tier)
        got = fn(theta, centres, mnorms, keys, pos, post_rope, p_now, offsets)
        assert np.max(np.abs(got - ref) / scale) < 1e-12, tier


@pytest.mark.parametrize("post_rope", [True, False])
@pytest.mark.parametrize("d,interleaved", [(64, False), (256, False), (128, True), (64, True)])
def test_identical_queries_logit_sum_other_layouts(post_rope, d, interleaved):
    """The textbook attention-logit special case for head dims 64/256 and interleaved pairs."""
    rng = np.random.default_rng(17 + d + interleaved)
    theta, G, nq = 1e4, 2, 3
    offsets = [1, 2, 4, 8, 16, 32, 64, 128]
    rope = rope_il_ld if interleaved else rope_ld
    pabs = pair_abs_il if interleaved else pair_abs
    qs = rng.standard_normal((G, d))
    cm = [oracle.calib(np.repeat(qs[g][None], nq, axis=0), interleaved=interleaved) for g in range(G)]
    centres = np.array([c for c, _ in cm])
    mnorms = np.array([m for _, m in cm])
    n = 12
    pos = rng.integers(0, 20000, size=n)
    p_now = 20000
    keys_pre = rng.standard_normal((n, d))
    keys = np.array([rope(keys_pre[j], pos[j], theta) for j in range(n)], dtype=np.float64) \
        if post_rope else keys_pre
    ref = np.array([float(_explicit_logit_sum(qs, keys[j], pos[j], post_rope, p_now, offsets, theta,
                                              rope)) for j in range(n)])
    scale = np.array([len(offsets) * np.mean([np.sum(pabs(q) * pabs(keys[j])) for q in qs])
                      for j in range(n)])
    for tier in ("literal", "collapsed", "absorbed"):
        fn = getattr(oracle, "score_" + tier)
        got = fn(theta, centres, mnorms, keys, pos, post_rope, p_now, offsets, interleaved=interleaved)
        assert np.max(np.abs(got - ref) / scale) < 1e-12, tier


@pytest.mark.parametrize("post_rope", [True, False])
def test_zero_centre_gives_norm_sum(post_rope):
    """Queries q and -q => qbar = 0, E|q_f| = |q_f|: score = (1/G) sum_g sum_f |q_f^g| |k_f|."""
    rng = np.random.default_rng(12)
    d, theta, G = 128, 1e6, 4
    qs = rng.standard_normal((G, d))
    cs, ms = zip(*[oracle.calib(np.stack([q, -q])) for q in qs])
    cs, ms = np.array(cs), np.array(ms)
    assert np.all(cs == 0.0)
    n = 16
    keys = rng.standard_normal((n, d))
    pos = rng.integers(0, 5000, size=n)
    ref = np.array([np.mean([np.sum(pair_abs(q) * pair_abs(keys[j])) for q in qs]) for j in range(n)])
    for fn in (oracle.score_literal, oracle.score_collapsed, oracle.score_absorbed):
        got = fn(theta, cs, ms, keys, pos, post_rope, 6000, [1, 2, 4])
        np.testing.assert_allclose(got, ref, rtol=1e-13)


def test_two_queries_trig_and_norm_parts():
    """Nq = 2 distinct queries: qbar = (q1+q2)/2, E|q_f| = (|q1_f|+|q2_f|)/2.  Trig part
    is the explicit logit sum of the averaged vector; norm part sum_f (E|q_f|-|qbar_f|)|k_f|."""
    rng = np.random.default_rng(13)
    d, theta = 128, 1e6
    offsets = [1, 2, 4, 8]
    q1, q2 = rng.standard_normal(d), rng.standard_normal(d)
    c, m = oracle.calib(np.stack([q1, q2]))
    qmean = (q1 + q2) / 2
    mexp = (pair_abs(q1) + pair_abs(q2)) / 2
    n = 10
    pos = rng.integers(0, 3000, size=n)
    keys_post = np.array([rope_ld(rng.standard_normal(d), pos[j], theta) for j in range(n)],
                         dtype=np.float64)
    ref = []
    for j in range(n):
        trig = float(_explicit_logit_sum([qmean], keys_post[j], pos[j], True, 3000, offsets, theta))
        norm = float(np.sum((mexp - pair_abs(qmean)) * pair_abs(keys_post[j])))
        ref.append(trig + norm)
    got = oracle.score_literal(theta, c[None], m[None], keys_post, pos, True, 3000, offsets)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------- tier agreement

@pytest.mark.parametrize("post_rope", [True, False])
@pytest.mark.parametrize("G,n_off", [(1, 13), (4, 13), (8, 17)])
def test_literal_collapsed_absorbed_agree(post_rope, G, n_off):
    rng = np.random.default_rng(100 + G + n_off)
    d, theta = 128, 1e6
    offsets = [2 ** e for e in range(n_off)]
    qs = rng.standard_normal((G, 64, d)) + 2 * rng.standard_normal((G, 1, d))
    cm = [oracle.calib(q) for q in qs]
    cs = np.array([c for c, _ in cm])
    ms = np.array([m for _, m in cm])
    n = 64
    keys = rng.standard_normal((n, d)) * np.exp(rng.standard_normal(d))
    pos = rng.integers(0, 131072, size=n)
    p_now = 131072
    a = oracle.score_literal(1e6, cs, ms, keys, pos, post_rope, p_now, offsets)
    b = oracle.score_collapsed(1e6, cs, ms, keys, pos, post_rope, p_now, offsets)
    c = oracle.score_absorbed(1e6, cs, ms, keys, pos, post_rope, p_now, offsets)
    scale = np.sum(np.abs(keys), axis=1) * np.max(np.abs(cs)) * n_off + 1.0
    assert np.max(np.abs(a - b) / scale) < 1e-12
    assert np.max(np.abs(a - c) / scale) < 1e-12


# ------------------------------------------------------------ invariances

def test_pre_rope_score_is_shift_invariant():
    rng = np.random.default_rng(21)
    d, G = 128, 2
    cs = rng.standard_normal((G, 64, 2))
    ms = np.hypot(cs[..., 0], cs[..., 1]) + rng.random((G, 64))
    keys = rng.standard_normal((20, d))
    pos = rng.integers(0, 8000, size=20)
    a = oracle.score_literal(1e6, cs, ms, keys, pos, False, 9000, [1, 2, 4, 8])
    b = oracle.score_literal(1e6, cs, ms, keys, pos + 50000, False, 59000, [1, 2, 4, 8])
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12 * np.max(np.abs(a)))


def test_score_scales_exactly_with_keys():
    rng = np.random.default_rng(22)
    cs = rng.standard_normal((2, 64, 2))
    ms = np.hypot(cs[..., 0], cs[..., 1]) + 0.3
    keys = rng.standard_normal((12, 128))
    pos = np.arange(12)
    for fn in (oracle.score_literal, oracle.score_absorbed):
        a = fn(1e6, cs, ms, keys, pos, True, 12, [1, 2, 4])
        b = fn(1e6, cs, ms, 4.0 * keys, pos, True, 12, [1, 2, 4])
        assert np.array_equal(4.0 * a, b)


# ------------------------------------------------------------- calibration

def test_calib_single_query():
    rng = np.random.default_rng(31)
    q = rng.standard_normal((1, 128))
    c, m = oracle.calib(q)
    np.testing.assert_array_equal(c[:, 0], q[0, :64])
    np.testing.assert_array_equal(c[:, 1], q[0, 64:])
    np.testing.assert_allclose(m, np.hypot(q[0, :64], q[0, 64:]), rtol=1e-15)


def test_calib_interleaved_pairs():
    """Interleaved layout: pair f is dims (2f, 2f+1)."""
    rng = np.random.default_rng(33)
    q = rng.standard_normal((500, 64)) + rng.standard_normal(64)
    c, m = oracle.calib(q, interleaved=True)
    np.testing.assert_allclose(c[:, 0], q[:, 0::2].mean(axis=0), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(c[:, 1], q[:, 1::2].mean(axis=0), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(m, np.hypot(q[:, 0::2], q[:, 1::2]).mean(axis=0), rtol=1e-13)


def test_calib_matches_numpy_and_triangle_inequality():
    rng = np.random.default_rng(32)
    q = rng.standard_normal((1000, 128)) + rng.standard_normal(128)
    c, m = oracle.calib(q)
    np.testing.assert_allclose(c[:, 0], q[:, :64].mean(axis=0), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(c[:, 1], q[:, 64:].mean(axis=0), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(m, np.hypot(q[:, :64], q[:, 64:]).mean(axis=0), rtol=1e-13)
    assert np.all(m >= np.hypot(c[:, 0], c[:, 1]))


# ----------------------------------------------------------------- select

def _kept_by_rank(s, B, W):
    """Brute force: slot j < N-W is kept iff fewer than B-W slots beat it."""
    n = len(s)
    if n <= B:
        return list(range(n))
    M, K = n - W, B - W
    kept = []
    for j in range(n):
        if j >= M:
            kept.append(j)
            continue
        beats = sum(1 for i in range(M) if s[i] > s[j] or (s[i] == s[j] and i > j))
        if beats < K:
            kept.append(j)
    return kept


def test_select_brute_force_tiny_rows():
    rng = np.random.default_rng(41)
    for n in list(range(0, 13)) + [17, 31, 40]:
        for trial in range(3):
            s = rng.integers(-3, 4, size=n).astype(np.float64)  # many ties
            if trial == 2:
                s = rng.standard_normal(n)
            for B in range(1, n + 3):
                for W in range(0, B + 1):
                    got = oracle.select(s, B, W)
                    assert list(got) == _kept_by_rank(s, B, W), (n, B, W, s)


def test_select_matches_lexsort_and_invariants():
    rng = np.random.default_rng(42)
    for n, B, W in [(4096, 512, 64), (5000, 2048, 128), (700, 699, 0), (1000, 300, 300)]:
        s = np.round(rng.standard_normal(n) * 50) / 4  # ties
        kept = oracle.select(s, B, W)
        M, K = n - W, B - W
        order = np.lexsort((-np.arange(M), -s[:M]))  # score desc, then slot desc
        ref = np.sort(np.concatenate([order[:K], np.arange(M, n)]))
        np.testing.assert_array_equal(kept, ref)
        assert len(kept) == min(n, B)
        assert np.all(np.diff(kept) > 0)
        assert set(range(n - W, n)) <= set(kept.tolist())
        ev = np.setdiff1d(np.arange(M), kept)
        kn = kept[kept < M]
        if len(ev) and len(kn):
            assert s[kn].min() >= s[ev].max()


def test_select_all_equal_keeps_most_recent():
    s = np.full(1000, 3.5)
    np.testing.assert_array_equal(oracle.select(s, 100, 10), np.arange(900, 1000))


def test_select_nan_ranks_last_and_bad_args():
    s = np.array([np.nan, 1.0, np.nan, -5.0, 2.0, 0.0])
    np.testing.assert_array_equal(oracle.select(s, 3, 1), [1, 4, 5])
    with pytest.raises(ValueError):
        oracle.select(s, 2, 3)
    with pytest.raises(ValueError):
        oracle.select(s, 0, 0)


# ----------------------------------------------------------------- gather

def test_gather_matches_fancy_indexing():
    rng = np.random.default_rng(51)
    src = rng.integers(0, 2**16, size=(300, 128)).astype(np.uint16)
    idx = np.sort(rng.choice(300, size=77, replace=False))
    np.testing.assert_array_equal(oracle.gather(src, idx), src[idx])
    np.testing.assert_array_equal(oracle.gather(src, np.arange(300)), src)
    p = rng.integers(0, 10**6, size=300).astype(np.int32)
    np.testing.assert_array_equal(oracle.gather(p, idx), p[idx])


def test_bf16_widening_is_exact():
    bits = np.array([0x3F80, 0xBF80, 0x0000, 0x8000, 0x7F7F, 0x0001, 0x4049], dtype=np.uint16)
    got = oracle.bf16_bits_to_f64(bits)
    assert got[0] == 1.0 and got[1] == -1.0 and got[2] == 0.0
    assert got[4] == float(np.float32(3.3895313892515355e38))
    assert got[5] == 2.0 ** -133
    assert got[6] == 3.140625


def test_e4m3_decoding_matches_definition_and_torch():
    import torch
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_bits_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref)) and np.isnan(got).sum() == 2
    np.testing.assert_array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])
    # hand-checked codes: 1.0, the largest finite 448, the smallest subnormal 2^-9, -2
    assert got[0x38] == 1.0 and got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0xC0] == -2.0


# ------------------------------------------------ online centres, diagnostics

def test_calib_online_equals_weighted_mean():
    """decay = 1: the plain mean of every query seen (numpy, one concatenation);
    decay < 1: numpy.average with weight decay^(batches after the query's own)."""
    rng = np.random.default_rng(51)
    d = 16
    batches = [rng.standard_normal((n, d)) + 1.5 for n in (5, 1, 7, 3)]
    q = np.concatenate(batches)
    F = d // 2
    c, m = oracle.calib_online(batches, 1.0)
    np.testing.assert_allclose(c[:, 0], q[:, :F].mean(axis=0), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(c[:, 1], q[:, F:].mean(axis=0), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(m, np.hypot(q[:, :F], q[:, F:]).mean(axis=0), rtol=1e-14)
    decay = 0.7
    w = np.concatenate([np.full(len(b), decay ** (len(batches) - 1 - i)) for i, b in enumerate(batches)])
    c, m = oracle.calib_online(batches, decay)
    np.testing.assert_allclose(c[:, 0], np.average(q[:, :F], axis=0, weights=w), rtol=1e-13)
    np.testing.assert_allclose(c[:, 1], np.average(q[:, F:], axis=0, weights=w), rtol=1e-13)
    np.testing.assert_allclose(m, np.average(np.hypot(q[:, :F], q[:, F:]), axis=0, weights=w), rtol=1e-13)
    ci, mi = oracle.calib_online(batches, decay, interleaved=True)
    np.testing.assert_allclose(ci[:, 1], np.average(q[:, 1::2], axis=0, weights=w), rtol=1e-13)
    np.testing.assert_allclose(mi, np.average(np.hypot(q[:, 0::2], q[:, 1::2]), axis=0, weights=w), rtol=1e-13)


@pytest.mark.parametrize("interleaved", [False, True])
def test_key_centres_undo_rope(interleaved):
    """Keys rotated by an explicit RoPE at random positions: their key centre is the
    numpy mean of the pre-RoPE pairs; a pre-RoPE cache needs no positions."""
    rng = np.random.default_rng(52 + interleaved)
    d, theta, n = 64, 1e4, 40
    pre = rng.standard_normal((n, d)) + 2.0
    pos = rng.integers(0, 200000, size=n)
    rope = rope_il_ld if interleaved else rope_ld
    post = np.array([rope(pre[j], pos[j], theta) for j in range(n)], dtype=np.float64)
    re, im = (pre[:, 0::2], pre[:, 1::2]) if interleaved else (pre[:, :d // 2], pre[:, d // 2:])
    for keys, post_rope in ((post, True), (pre, False)):
        c, m = oracle.key_centres(theta, keys, pos, post_rope, interleaved)
        np.testing.assert_allclose(c[:, 0], re.mean(axis=0), rtol=0, atol=1e-12 * np.abs(re).max())
        np.testing.assert_allclose(c[:, 1], im.mean(axis=0), rtol=0, atol=1e-12 * np.abs(im).max())
        np.testing.assert_allclose(m, np.hypot(re, im).mean(axis=0), rtol=1e-12)
    c, m = oracle.key_centres(theta, np.zeros((0, d)), np.zeros(0), True, interleaved)
    assert np.all(c == 0) and np.all(m == 0)


def test_calib_stats_closed_forms():
    # one pair: centre 3+4i (|c| = 5), mean norm 10 -> concentration 1/2
    conc, (hc, drift) = oracle.calib_stats(np.array([[3.0, 4.0]]), np.array([10.0]))
    assert conc[0] == 0.5 and hc == 0.5 and drift == 0.0
    # drift against centre 0, norm 5: (|3+4i - 0| + |10 - 5|) / 5 = 2
    _, (_, drift) = oracle.calib_stats(np.array([[3.0, 4.0]]), np.array([10.0]), np.zeros((1, 2)), np.array([5.0]))
    assert drift == 2.0
    # all queries identical: every pair fully concentrated; q and -q: none
    rng = np.random.default_rng(53)
    q = rng.standard_normal(32)
    c, m = oracle.calib(np.stack([q, q, q]))
    conc, (hc, drift) = oracle.calib_stats(c, m, c, m)
    np.testing.assert_allclose(conc, 1.0, rtol=1e-15)
    assert abs(hc - 1.0) < 1e-15 and drift == 0.0
    c, m = oracle.calib(np.stack([q, -q]))
    conc, (hc, _) = oracle.calib_stats(c, m)
    assert np.all(conc == 0.0) and hc == 0.0
    # a zero-norm pair reports 0, not NaN
    conc, (hc, _) = oracle.calib_stats(np.zeros((2, 2)), np.zeros(2))
    assert np.all(conc == 0.0) and hc == 0.0


# ------------------------------------------------------- decode attention

def test_attention_matches_torch_sdpa_and_closed_forms():
    import torch
    rng = np.random.default_rng(61)
    d = 64
    for n in (1, 2, 7, 300):
        q = rng.standard_normal(d)
        k = rng.standard_normal((n, d)) * 0.7
        v = rng.standard_normal((n, d))
        scale = 1.0 / np.sqrt(d)
        out, lse = oracle.attention(q, k, v, scale)
        tq, tk, tv = (torch.from_numpy(x).to(torch.float64) for x in (q[None, None, None], k[None, None], v[None, None]))
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale)[0, 0, 0].numpy()
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)
        s = scale * (k @ q)
        np.testing.assert_allclose(lse, np.log(np.sum(np.exp(s))), rtol=1e-13)
    # q = 0: every weight equal -> mean of V, lse = log n
    v = rng.standard_normal((5, d))
    out, lse = oracle.attention(np.zeros(d), rng.standard_normal((5, d)), v, 1.0)
    np.testing.assert_allclose(out, v.mean(axis=0), rtol=1e-14)
    assert abs(lse - np.log(5.0)) < 1e-15
    # two keys: out = sigmoid(s1 - s2) v1 + sigmoid(s2 - s1) v2
    q = np.zeros(d)
    q[0] = 1.0
    k = np.zeros((2, d))
    k[0, 0], k[1, 0] = 2.0, -1.0
    v = rng.standard_normal((2, d))
    out, lse = oracle.attention(q, k, v, 1.0)
    w1 = 1.0 / (1.0 + np.exp(-3.0))
    np.testing.assert_allclose(out, w1 * v[0] + (1 - w1) * v[1], rtol=1e-14)
    assert abs(lse - np.log(np.exp(2.0) + np.exp(-1.0))) < 1e-14
    # huge scores do not overflow (the maximum is subtracted first)
    out, lse = oracle.attention(q, 1000.0 * k, v, 1.0)
    np.testing.assert_allclose(out, v[0], rtol=1e-14)
    assert abs(lse - 2000.0) < 1e-12
    # empty row
    out, lse = oracle.attention(q, np.zeros((0, d)), np.zeros((0, d)), 1.0)
    assert np.all(out == 0) and lse == -np.inf
