"""tri_score_noalloc: tri_score for callers that cannot allocate device memory
(code inside another framework's memory pool, plugins whose host process owns
every allocation, serving loops that allocate only at start-up).  Its scratch
is a fixed array inside the library instead of a caller workspace.

The entry point runs the same kernels in the same order as tri_score, so its
scores must equal tri_score's (with a workspace) bit for bit on the same inputs,
call after call on the shared scratch: a larger call, then a smaller one on
another cache, then the largest the scratch allows (TRI_NOALLOC_MAX_ROWS rows at
head dim 256).  Against the oracle the scores meet the parity tests' tolerance
(1e-4 of the series bound).  Sizes above the fixed scratch are rejected before
any launch.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import kv_cache_compression_calib_b200 as tri
import synth
from kv_cache_compression_calib_b200 import _abi
from tests import harness as H
from tests.test_gpu_parity import model_of, oracle_centres, oracle_scores, to_dev

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _noalloc_abi(m, kv, K, pos, c, n, p_now, offsets, mode, scores):
    """Call the entry point directly through the C ABI."""
    L = _abi.load()
    offs = (ctypes.c_int32 * len(offsets))(*offsets)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.tri_score_noalloc(ctypes.byref(m), ctypes.byref(kv), K.data_ptr(),
                               pos.data_ptr() if pos is not None else None, c.data_ptr(),
                               n.data_ptr(), p_now.data_ptr(), offs, len(offsets), mode,
                               scores.data_ptr(), stream)


def _both(dev, cs, ms, mode):
    """(tri_score with a workspace, tri_score_noalloc) scores on one device cache;
    the no-alloc output starts as NaN so an unwritten score cannot pass."""
    wl = dev.wl
    m = model_of(wl, len(dev.layers))
    S = len(dev.lens)
    kv = tri.kv_contig(S, dev.row_off, dev.total, tri.elem_type_of(dev.K))
    c = torch.tensor(cs, dtype=torch.float32, device=DEV)
    n = torch.tensor(ms, dtype=torch.float32, device=DEV)
    n_out = max(dev.total, 1)
    ref = torch.full((n_out,), float("nan"), dtype=torch.float32, device=DEV)
    ws = tri.alloc_workspace(m, S, 1)
    tri.tri_score(m, kv, dev.K, dev.pos, c, n, dev.p_now, wl.offsets, mode, ref, ws)
    got = torch.full((n_out,), float("nan"), dtype=torch.float32, device=DEV)
    assert _noalloc_abi(m, kv, dev.K, dev.pos, c, n, dev.p_now, wl.offsets, mode, got) == 0
    torch.cuda.synchronize()
    st, flags = tri.tri_status_check(ws)
    assert st == 0 and flags == 0
    return ref[:dev.total].cpu(), got[:dev.total].cpu()


def _assert_bits_equal(ref, got):
    assert torch.equal(ref.view(torch.int32), got.view(torch.int32))


def test_noalloc_equals_workspace_scoring_call_after_call():
    base = synth.WORKLOADS["single_layer_4k"].with_(n_calib=64)
    cases = [
        # the larger call first (6 rows more than the next one), pre-RoPE keys
        (base.with_(name="noalloc1", n_layers=2, batch=3), [900, 33, 2500], False, tri.TRI_KEYS_PRE_ROPE),
        # then fewer rows on another cache, post-RoPE keys
        (base.with_(name="noalloc2"), [1537], True, tri.TRI_KEYS_POST_ROPE),
        # and the larger shape once more, after the smaller one
        (base.with_(name="noalloc3", n_layers=2, batch=3), [64, 4096, 7], True, tri.TRI_KEYS_POST_ROPE),
    ]
    for wl, lens, rotate, mode in cases:
        host = synth.make_contig(wl, "cpu", lens=lens, rotate=rotate)
        cs, ms = oracle_centres(host)
        ref, got = _both(to_dev(host), cs, ms, mode)
        _assert_bits_equal(ref, got)
        oref, bound = oracle_scores(host, cs, ms, post_rope=rotate, tier="collapsed")
        assert H.score_error(got.numpy().astype(np.float64), oref, bound) <= 1e-4


def test_noalloc_at_the_row_limit_with_the_largest_head_dim():
    """TRI_NOALLOC_MAX_ROWS rows (16 layers x 32 sequences x 8 KV heads) at head
    dim 256, so every byte of the scratch's coefficient area is written; short
    rows of 0 to 9 keys keep the oracle check quick."""
    rows = _abi.TRI_NOALLOC_MAX_ROWS
    L, S = 16, 32
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="noallocmax", n_layers=L, batch=S, head_dim=256,
                                                  theta=1e4, n_calib=8)
    assert L * S * wl.n_kv_heads == rows
    lens = [int(x) for x in np.random.default_rng(7).integers(0, 10, size=S)]
    host = synth.make_contig(wl, "cpu", lens=lens, rotate=True)
    cs, ms = oracle_centres(host)
    ref, got = _both(to_dev(host), cs, ms, tri.TRI_KEYS_POST_ROPE)
    _assert_bits_equal(ref, got)
    sample = [0, 1, rows // 2, rows - 2, rows - 1]
    oref, bound = oracle_scores(host, cs, ms, post_rope=True, tier="collapsed", rows=sample)
    keep = ~np.isnan(oref)
    assert keep.any()
    assert H.score_error(got.numpy().astype(np.float64)[keep], oref[keep], bound[keep]) <= 1e-4


def test_noalloc_rejects_rows_beyond_scratch():
    m = tri.model(_abi.TRI_NOALLOC_MAX_ROWS // 8 + 1, 32, 8, 1e6)
    ro = torch.zeros(m.n_layers * 8 + 1, dtype=torch.int64, device=DEV)
    kv = tri.kv_contig(1, ro, 0)
    dummy = torch.zeros(16, device=DEV)
    st = _noalloc_abi(m, kv, dummy, None, dummy, dummy, ro, [1, 2], tri.TRI_KEYS_POST_ROPE, dummy)
    assert st == _abi.TRI_ERR_WORKSPACE_TOO_SMALL
