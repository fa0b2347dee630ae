"""Compaction with V and the outputs in pinned host memory: the gather reads the
kept records of V over the host link and writes the compacted cache straight to
host memory.  The results must equal, bit for bit, those of the same call with
everything on the device, for the two-call path and the fused one."""
import numpy as np
import pytest
import torch

import kv_cache_compression_calib_b200 as tri
import synth
from tests import harness as H
from tests.test_gpu_parity import POST, gpu_compact, gpu_score, model_of, oracle_centres, to_dev

pytestmark = pytest.mark.gpu
DEV = "cuda"


def host_compact(cache, scores, B, W, fused_max_row=None, centres=None):
    wl = cache.wl
    m = model_of(wl, len(cache.layers))
    S, R = len(cache.lens), cache.n_rows
    kv = tri.kv_contig(S, cache.row_off, cache.total, tri.elem_type_of(cache.K))
    ws = tri.alloc_workspace(m, S, B)
    hV = cache.V.cpu().pin_memory()
    Ko = torch.zeros(R, B, wl.head_dim, dtype=cache.K.dtype).pin_memory()
    Vo = torch.zeros(R, B, wl.head_dim, dtype=cache.K.dtype).pin_memory()
    po = torch.full((R, B), -7, dtype=torch.int32).pin_memory()
    kept = torch.full((R, B), -1, dtype=torch.int32, device=DEV)
    cnt = torch.full((R,), -1, dtype=torch.int32, device=DEV)
    if fused_max_row is None:
        tri.tri_compact(m, kv, scores, B, W, cache.K, hV, cache.pos, tri.out_contig(), Ko, Vo, po, kept, cnt, ws)
    else:
        c32, m32 = centres
        tri.tri_score_compact(m, kv, cache.K, hV, cache.pos, c32, m32, cache.p_now, wl.offsets, POST, B, W,
                              fused_max_row, tri.out_contig(), Ko, Vo, po, kept, cnt, None, ws)
    st, flags = tri.tri_status_check(ws)
    torch.cuda.synchronize()
    return dict(K=Ko.clone(), V=Vo.clone(), pos=po.clone(), kept=kept.cpu().numpy(), cnt=cnt.cpu().numpy(),
                status=st, flags=flags)


@pytest.mark.parametrize("fused", [False, True])
def test_pinned_host_records_equal_the_device_path(fused):
    wl = synth.WORKLOADS["single_layer_4k"].with_(name="hostrec", batch=3, n_calib=32)
    host = synth.make_contig(wl, "cpu", lens=[4096, 700, 33])
    cs, ms = oracle_centres(host)
    dev = to_dev(host)
    B, W = 512, 64
    scores = gpu_score(dev, cs, ms, B=B)
    ref = gpu_compact(dev, scores, B, W)
    c32 = torch.tensor(cs, dtype=torch.float32, device=DEV)
    m32 = torch.tensor(ms, dtype=torch.float32, device=DEV)
    got = host_compact(dev, scores, B, W, fused_max_row=4096 if fused else None, centres=(c32, m32))
    assert got["status"] == 0 and got["flags"] == 0
    np.testing.assert_array_equal(got["kept"], ref["kept"])
    np.testing.assert_array_equal(got["cnt"], ref["cnt"])
    for r in range(host.n_rows):
        n = int(ref["cnt"][r])
        assert torch.equal(H.torch_bits(got["K"][r, :n]), H.torch_bits(ref["K"][r, :n]))
        assert torch.equal(H.torch_bits(got["V"][r, :n]), H.torch_bits(ref["V"][r, :n]))
        assert torch.equal(got["pos"][r, :n], ref["pos"][r, :n])
