"""Selection and compaction of rows longer than one 32768-slot chunk of the
selection kernel ("TriAttention：基于三角函数 KV 压缩的高效长推理", 流程详解 step 4),
with special scores: exact ties, NaN, infinities, signed zeros, subnormals,
outliers, a tie block across the 32768-slot chunk boundary, and samples that
force the key-space bin map.  Given the same fp32 scores, the kept slots must
equal oracle.select and the compacted K, V and positions oracle.gather, bit for
bit.

The cache is one layer of single-head rows with random record bits (head dim
64): the selection and the gather only move bits, so the keys need no
structure here.
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_calib_b200 as tri
import oracle
from tests import harness as H
from tests.test_gpu_parity import _scores_case

pytestmark = pytest.mark.gpu
DEV = "cuda"
CHUNK = 32768
D = 64


class LongRows:
    """Rows of the given lengths (one layer, one KV head, one sequence per row)."""

    def __init__(self, lens, seed=11):
        self.lens = np.asarray(lens, dtype=np.int64)
        self.row_off_np = np.concatenate([[0], np.cumsum(self.lens)]).astype(np.int64)
        self.total = int(self.row_off_np[-1])
        self.n_rows = len(lens)
        g = torch.Generator().manual_seed(seed)
        self.K = torch.randint(-32768, 32767, (self.total, D), dtype=torch.int16, generator=g).view(torch.bfloat16)
        self.V = torch.randint(-32768, 32767, (self.total, D), dtype=torch.int16, generator=g).view(torch.bfloat16)
        self.pos = torch.cat([torch.arange(int(n), dtype=torch.int32) for n in self.lens])
        self.dK, self.dV, self.dpos = self.K.to(DEV), self.V.to(DEV), self.pos.to(DEV)
        self.row_off = torch.as_tensor(self.row_off_np, device=DEV)

    def compact(self, scores32, B, W):
        m = tri.model(1, self.n_rows, self.n_rows, 1e6, head_dim=D)  # one sequence, n_rows KV heads
        kv = tri.kv_contig(1, self.row_off, self.total)
        ws = tri.alloc_workspace(m, 1, B)
        R = self.n_rows
        Ko = torch.zeros(R, B, D, dtype=torch.bfloat16, device=DEV)
        Vo = torch.zeros_like(Ko)
        po = torch.full((R, B), -7, dtype=torch.int32, device=DEV)
        kept = torch.full((R, B), -1, dtype=torch.int32, device=DEV)
        cnt = torch.full((R,), -1, dtype=torch.int32, device=DEV)
        s = torch.tensor(scores32, dtype=torch.float32, device=DEV)
        tri.tri_compact(m, kv, s, B, W, self.dK, self.dV, self.dpos, tri.out_contig(), Ko, Vo, po, kept, cnt, ws)
        st, flags = tri.tri_status_check(ws)
        return dict(K=Ko.cpu(), V=Vo.cpu(), pos=po.cpu(), kept=kept.cpu().numpy(), cnt=cnt.cpu().numpy(),
                    status=st, flags=flags)

    def check_exact(self, res, scores32, B, W):
        Kb, Vb = H.raw_bits(self.K), H.raw_bits(self.V)
        pos = self.pos.numpy()
        Kob, Vob = H.raw_bits(res["K"]), H.raw_bits(res["V"])
        for r in range(self.n_rows):
            a, b = self.row_off_np[r], self.row_off_np[r + 1]
            ref = oracle.select(scores32[a:b], B, W)
            n = len(ref)
            assert res["cnt"][r] == n
            np.testing.assert_array_equal(res["kept"][r, :n], ref, err_msg=f"row {r} ({b - a} slots)")
            np.testing.assert_array_equal(Kob[r, :n], oracle.gather(Kb[a:b], ref))
            np.testing.assert_array_equal(Vob[r, :n], oracle.gather(Vb[a:b], ref))
            np.testing.assert_array_equal(res["pos"][r, :n].numpy(), oracle.gather(pos[a:b], ref))
            assert np.all(res["kept"][r, n:] == -1)


# Rows whose candidate slots (N - W) span 2, 3 and 5 chunks at W <= 256, and one
# of exactly 4 full chunks plus the window.
LONG_LENS = [CHUNK + 257, 70000, 131072, 4 * CHUNK + 256]


@pytest.fixture(scope="module")
def long_rows():
    return LongRows(LONG_LENS)


def _row_scores(rows, fn):
    out = np.empty(rows.total)
    for r in range(rows.n_rows):
        a, b = rows.row_off_np[r], rows.row_off_np[r + 1]
        out[a:b] = fn(r, b - a)
    return H.as_f32_exact(out)


@pytest.mark.parametrize("B,W", [(4096, 256), (2048, 128), (100, 0)])
@pytest.mark.parametrize("kind", ["all_equal", "quantized", "signed_zero", "nan", "wide", "inf",
                                  "subnormal", "huge", "straddle", "outlier"])
def test_long_rows_special_scores(long_rows, kind, B, W):
    rng = np.random.default_rng(17)
    s32 = _row_scores(long_rows, lambda r, n: _scores_case(kind, n, rng))
    res = long_rows.compact(s32, B, W)
    long_rows.check_exact(res, s32, B, W)
    if kind == "nan":
        assert res["flags"] & tri.TRI_FLAG_NONFINITE
    else:
        assert res["status"] == 0


@pytest.mark.parametrize("B,W", [(4096, 256), (2048, 128)])
def test_tie_block_across_the_chunk_boundary(long_rows, B, W):
    """K = B - W keys must come from the candidates: 60% of K sit well above, and
    a block of 2K exactly equal scores straddles slot 32768 (and, in longer rows,
    slots 65536 and 98304), so the threshold is that value and the kept ties are
    the most recent ones, counted across chunks."""
    K = B - W

    def fn(r, n):
        rng = np.random.default_rng(100 + r)
        s = rng.standard_normal(n) - 10.0
        hi = rng.choice(n - W, size=int(0.6 * K), replace=False)
        s[hi] = 50.0 + rng.random(len(hi))
        for c in (CHUNK, 2 * CHUNK, 3 * CHUNK):
            if c < n - W:  # the block ends at the last candidate slot at most
                blk = np.arange(c - K, min(c + K, n - W))
                blk = blk[s[blk] < 50.0]
                s[blk] = 7.0
        return s

    s32 = _row_scores(long_rows, fn)
    res = long_rows.compact(s32, B, W)
    assert res["status"] == 0
    long_rows.check_exact(res, s32, B, W)


def _sample_slots(M):
    """The evenly spaced sample the selection kernel reads first (1024 slots of M)."""
    return (np.arange(1024, dtype=np.int64) * M) // 1024


@pytest.mark.parametrize("sample", ["constant", "nan", "inf"])
def test_key_space_map_on_multi_chunk_rows(long_rows, sample):
    """A sample with no usable value range (every sampled score equal, one NaN,
    or an infinity) makes the kernel bin by key space over the whole row."""
    B, W = 4096, 256

    def fn(r, n):
        rng = np.random.default_rng(200 + r)
        s = rng.standard_normal(n) * 3.0
        idx = _sample_slots(n - W)
        if sample == "constant":
            s[idx] = 0.25
        elif sample == "nan":
            s[idx[::97]] = np.nan
        else:
            s[idx[5]] = -np.inf
            s[idx[700]] = np.inf
        return s

    s32 = _row_scores(long_rows, fn)
    res = long_rows.compact(s32, B, W)
    long_rows.check_exact(res, s32, B, W)
    if sample == "nan":
        assert res["flags"] & tri.TRI_FLAG_NONFINITE
    else:
        assert res["status"] == 0


def _sampled(n, W):
    """Slots the first pass samples on a row of n slots with window W (the runs
    of 8 starting at (t * (n - W) / 512) rounded down to a multiple of 8)."""
    M = n - W
    starts = ((np.arange(512, dtype=np.int64) * M) // 512) & ~7
    return (starts[:, None] + np.arange(8)).ravel()


@pytest.mark.parametrize("case", ["fine_ties", "specials_off_sample", "negative"])
def test_band_cases_on_long_rows(long_rows, case):
    """Scores whose sample gives a usable band, so the single-pass selection
    decides: many exact ties near the threshold (scores on a 0.01 grid), NaN,
    +-inf and -0.0 at slots the sample does not read, and all-negative scores."""
    def fn(r, n):
        rng = np.random.default_rng(300 + r)
        if case == "fine_ties":
            return np.round(rng.standard_normal(n) * 3.0, 2)
        if case == "negative":
            return -np.abs(rng.standard_normal(n)) - 5.0
        s = rng.standard_normal(n)
        off = np.setdiff1d(np.arange(n), _sampled(n, 256))
        pick = rng.choice(off, size=40, replace=False)
        s[pick[:10]] = np.nan
        s[pick[10:20]] = np.inf
        s[pick[20:30]] = -np.inf
        s[pick[30:]] = -0.0
        return s

    for B, W in ((4096, 256), (1024, 0)):
        s32 = _row_scores(long_rows, fn)
        res = long_rows.compact(s32, B, W)
        long_rows.check_exact(res, s32, B, W)
        if case == "specials_off_sample":
            assert res["flags"] == tri.TRI_FLAG_NONFINITE
        else:
            assert res["status"] == 0


@pytest.mark.parametrize("d,elem", [(64, "fp8"), (128, "fp8"), (256, "bf16")])
@pytest.mark.parametrize("paged_out", [False, True])
def test_long_row_copy_record_sizes_and_paged_output(d, elem, paged_out):
    """The select-and-gather kernel copies a long row's kept records through its
    shared memory in groups whose size depends on the record (64, 128 and 512
    bytes here; 128 above): K, V and positions bit for bit, into [R][B] or into a
    fresh, shuffled paged block table."""
    lens = np.array([CHUNK + 4000, 90000])
    R, B, W, bs = len(lens), 4096, 256, 16
    row_off_np = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    total = int(row_off_np[-1])
    g = torch.Generator().manual_seed(23)
    if elem == "fp8":
        K = torch.randint(0, 256, (total, d), dtype=torch.uint8, generator=g).view(torch.float8_e4m3fn)
        V = torch.randint(0, 256, (total, d), dtype=torch.uint8, generator=g).view(torch.float8_e4m3fn)
    else:
        K = torch.randint(-32768, 32767, (total, d), dtype=torch.int16, generator=g).view(torch.bfloat16)
        V = torch.randint(-32768, 32767, (total, d), dtype=torch.int16, generator=g).view(torch.bfloat16)
    pos = torch.cat([torch.arange(int(n), dtype=torch.int32) for n in lens])
    rng = np.random.default_rng(29)
    s32 = H.as_f32_exact(rng.standard_normal(total))
    m = tri.model(1, R, R, 1e6, head_dim=d)  # one sequence, R KV heads
    kv = tri.kv_contig(1, torch.as_tensor(row_off_np, device=DEV), total, tri.elem_type_of(K))
    ws = tri.alloc_workspace(m, 1, B)
    kept = torch.full((R, B), -1, dtype=torch.int32, device=DEV)
    if paged_out:
        n_out = B // bs
        out_tbl = rng.permutation(n_out).reshape(1, n_out).astype(np.int32)
        Ko = torch.zeros(1, n_out, bs, R, d, dtype=K.dtype, device=DEV)
        po = torch.full((1, n_out, bs, R), -7, dtype=torch.int32, device=DEV)
        out = tri.out_paged(torch.as_tensor(out_tbl, device=DEV), bs, n_out)
    else:
        Ko = torch.zeros(R, B, d, dtype=K.dtype, device=DEV)
        po = torch.full((R, B), -7, dtype=torch.int32, device=DEV)
        out = tri.out_contig()
    Vo = torch.zeros_like(Ko)
    tri.tri_compact(m, kv, torch.tensor(s32, dtype=torch.float32, device=DEV), B, W, K.to(DEV), V.to(DEV),
                    pos.to(DEV), out, Ko, Vo, po, kept, None, ws)
    st, flags = tri.tri_status_check(ws)
    assert st == 0, flags
    Kb, Vb = H.raw_bits(K), H.raw_bits(V)
    Kob, Vob, pob = H.raw_bits(Ko.cpu()), H.raw_bits(Vo.cpu()), po.cpu().numpy()
    kept = kept.cpu().numpy()
    for r in range(R):
        a, b = row_off_np[r], row_off_np[r + 1]
        ref = oracle.select(s32[a:b], B, W)
        np.testing.assert_array_equal(kept[r], ref)
        i = np.arange(B)
        if paged_out:
            blk = out_tbl[0, i // bs]
            got_k, got_v, got_p = Kob[0, blk, i % bs, r], Vob[0, blk, i % bs, r], pob[0, blk, i % bs, r]
        else:
            got_k, got_v, got_p = Kob[r], Vob[r], pob[r]
        np.testing.assert_array_equal(got_k, oracle.gather(Kb[a:b], ref))
        np.testing.assert_array_equal(got_v, oracle.gather(Vb[a:b], ref))
        np.testing.assert_array_equal(got_p, oracle.gather(pos.numpy()[a:b], ref))
