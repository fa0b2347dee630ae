"""Failure detection on the GPU without a fault: the bounded wait of the staged
kernels is made to run out (a barrier nothing completes), and the host reads the
status it leaves; the context is then used again."""
import time

import numpy as np
import pytest
import torch

import kv_cache_compression_calib_b200 as tri
import synth
from tests import harness as H
from tests.test_gpu_parity import PRE, gpu_score, oracle_centres, oracle_scores, to_dev

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_staged_wait_times_out_and_the_context_stays_usable():
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    limit_ns = 20_000_000  # 20 ms
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    tri.tri_selftest_wait_timeout(ws, limit_ns)
    st, flags = tri.tri_status_check(ws)
    elapsed = time.perf_counter() - t0
    assert st == tri._abi.TRI_ERR_DEVICE_FLAG and flags == tri.TRI_FLAG_STAGE_TIMEOUT
    assert elapsed >= limit_ns * 1e-9
    st, flags = tri.tri_status_check(ws)  # the flag word was cleared
    assert st == 0 and flags == 0
    # the context still works: a staged scoring call meets the oracle
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="after", batch=2, n_calib=32)
    host = synth.make_contig(wl, "cpu", lens=[700, 129], rotate=False)
    cs, ms = oracle_centres(host)
    got = gpu_score(to_dev(host), cs, ms, key_mode=PRE).cpu().numpy().astype(np.float64)
    ref, bound = oracle_scores(host, cs, ms, post_rope=False, tier="collapsed")
    assert H.score_error(got[:host.total], ref, bound) <= 1e-4
