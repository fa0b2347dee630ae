"""tri_score_noalloc: tri_score for callers that cannot allocate device memory
(code inside another framework's memory pool, plugins whose host process owns
every allocation, serving loops that allocate only at start-up).  Its scratch
is a fixed array inside the library instead of a caller workspace.

Two calls in a row, on different caches, must give the scores of tri_score
(with a workspace) on the same inputs, within the score tolerance used by the
parity tests (1e-4 of the series bound); sizes above the fixed scratch are
rejected before any launch.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import kv_cache_compression_calib_b200 as tri
import synth
from kv_cache_compression_calib_b200 import _abi
from tests import harness as H

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(wl, lens, rotate):
    host = synth.make_contig(wl, "cpu", lens=lens, rotate=rotate)
    cs, ms = H.oracle_calibration(host.qcal)
    return host, H.as_f32_exact(cs), H.as_f32_exact(ms)


def _noalloc_abi(m, kv, K, pos, c, n, p_now, offsets, mode, scores):
    """Call the entry point directly through the C ABI."""
    L = _abi.load()
    offs = (ctypes.c_int32 * len(offsets))(*offsets)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.tri_score_noalloc(ctypes.byref(m), ctypes.byref(kv), K.data_ptr(),
                               pos.data_ptr() if pos is not None else None, c.data_ptr(),
                               n.data_ptr(), p_now.data_ptr(), offs, len(offsets), mode,
                               scores.data_ptr(), stream)


def test_noalloc_matches_workspace_scoring_twice():
    base = synth.WORKLOADS["single_layer_4k"].with_(n_calib=64)
    cases = [
        (base, None, True, tri.TRI_KEYS_POST_ROPE),
        (base.with_(name="noalloc2", n_layers=2, batch=3), [900, 33, 2500], False,
         tri.TRI_KEYS_PRE_ROPE),
    ]
    for wl, lens, rotate, mode in cases:
        host, cs, ms = _case(wl, lens, rotate)
        L = len(host.layers)
        m = tri.model(L, wl.n_q_heads, wl.n_kv_heads, wl.theta)
        S = len(host.lens)
        ro = host.row_off.to(DEV)
        kv = tri.kv_contig(S, ro, host.total)
        K, pos, pn = host.K.to(DEV), host.pos.to(DEV), host.p_now.to(DEV)
        c = torch.tensor(cs, dtype=torch.float32, device=DEV)
        n = torch.tensor(ms, dtype=torch.float32, device=DEV)
        ref = torch.empty(host.total, dtype=torch.float32, device=DEV)
        ws = tri.alloc_workspace(m, S, 1)
        tri.tri_score(m, kv, K, pos, c, n, pn, wl.offsets, mode, ref, ws)
        got = torch.full((host.total,), float("nan"), dtype=torch.float32, device=DEV)
        assert _noalloc_abi(m, kv, K, pos, c, n, pn, wl.offsets, mode, got) == 0
        torch.cuda.synchronize()
        ref, got = ref.cpu().numpy().astype(np.float64), got.cpu().numpy().astype(np.float64)
        Kf = H.to_f64(host.K)
        for r in range(host.n_rows):
            li, s, h = host.row_lhs(r)
            a, b = host.row_off_np[r], host.row_off_np[r + 1]
            bd = H.series_bound(wl.theta, cs[li], ms[li], h, wl.group, Kf[a:b], wl.offsets)
            assert H.score_error(got[a:b], ref[a:b], bd) <= 1e-4


def test_noalloc_rejects_rows_beyond_scratch():
    m = tri.model(_abi.TRI_NOALLOC_MAX_ROWS // 8 + 1, 32, 8, 1e6)
    ro = torch.zeros(m.n_layers * 8 + 1, dtype=torch.int64, device=DEV)
    kv = tri.kv_contig(1, ro, 0)
    dummy = torch.zeros(16, device=DEV)
    st = _noalloc_abi(m, kv, dummy, None, dummy, dummy, ro, [1, 2], tri.TRI_KEYS_POST_ROPE, dummy)
    assert st == _abi.TRI_ERR_WORKSPACE_TOO_SMALL
