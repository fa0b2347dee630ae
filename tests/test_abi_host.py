"""The C ABI without a GPU: the library loads, exports every symbol that
include/tri.h declares, and rejects bad arguments on the host before any
CUDA call (these calls never reach the device)."""
import ctypes
import os
import re

import pytest
import torch

import kv_cache_compression_calib_b200 as tri
from kv_cache_compression_calib_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tri.h")


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tri_[a-z_]+)\s*\(", src)))


def test_header_declares_the_abi():
    names = header_functions()
    assert names == sorted(_abi.EXPORTS)
    assert {"tri_calib", "tri_score", "tri_compact"} <= set(names)


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(tri.library_path())
    for name in header_functions():
        assert hasattr(L, name), name


def test_status_strings_and_version():
    L = _abi.load()
    for code, name in [(0, "TRI_OK"), (1, "TRI_ERR_INVALID_ARG"), (2, "TRI_ERR_UNSUPPORTED"),
                       (3, "TRI_ERR_ALIGNMENT"), (4, "TRI_ERR_WORKSPACE_TOO_SMALL"),
                       (5, "TRI_ERR_CUDA"), (6, "TRI_ERR_DEVICE_FLAG")]:
        assert L.tri_status_str(code).decode() == name
    assert tri.version() >= 1


def test_workspace_size():
    m = tri.model(36, 32, 8, 1e6)
    n = tri.tri_workspace_size(m, 1, 2048)
    R = 36 * 8
    assert n >= R * 768 + R * 2048 * 4 and n % 256 == 0
    assert tri.tri_workspace_size(m, 0, 2048) == 0
    assert tri.tri_workspace_size(m, 1, 0) == 0
    assert tri.tri_workspace_size(tri.model(1, 32, 8, 1e6, head_dim=96), 1, 16) == 0
    assert tri.tri_workspace_size(tri.model(1, 32, 8, 1e6, rope_style=2), 1, 16) == 0
    # per-row coefficients: 3 floats per pair, d/2 pairs
    for d in (64, 128, 256):
        md = tri.model(36, 32, 8, 1e6, head_dim=d, rope_style=tri.TRI_ROPE_INTERLEAVED)
        assert tri.tri_workspace_size(md, 1, 2048) >= R * 6 * d + R * 2048 * 4


# Fake (never dereferenced) device addresses: the host checks run first.
A = 1 << 20  # 1 MiB: aligned for every check


def _kv(layout=0, n_seqs=1, total=4096, row_off=A, table=None, max_blocks=0, bs=0, nb=0):
    return _abi.TriKvDesc(layout, n_seqs, total, row_off, table, max_blocks, bs, nb)


def _score(m, kv, K=A, pos=None, c=A, mn=A, pnow=A, offs=(1, 2, 4), mode=0, scores=A, ws=A,
           ws_bytes=1 << 30):
    L = _abi.load()
    arr = (ctypes.c_int32 * max(len(offs), 1))(*offs)
    return L.tri_score(ctypes.byref(m), ctypes.byref(kv) if kv is not None else None, K, pos, c, mn,
                       pnow, arr, len(offs), mode, scores, ws, ws_bytes, None)


def _compact(m, kv, B=64, W=8, scores=A, K=A, V=2 * A, pos=None, out=None, Ko=3 * A, Vo=4 * A,
             poso=None, kept=None, cnt=None, ws=A, ws_bytes=1 << 30):
    L = _abi.load()
    out = out or _abi.TriOutDesc(0, 0, None, 0, 0, 0)
    return L.tri_compact(ctypes.byref(m), ctypes.byref(kv), scores, B, W, K, V, pos, ctypes.byref(out),
                         Ko, Vo, poso, kept, cnt, ws, ws_bytes, None)


M = tri.model(1, 32, 8, 1e6)


@pytest.mark.parametrize("kwargs,status", [
    (dict(K=None), _abi.TRI_ERR_INVALID_ARG),
    (dict(scores=None), _abi.TRI_ERR_INVALID_ARG),
    (dict(offs=()), _abi.TRI_ERR_INVALID_ARG),
    (dict(offs=tuple(range(65))), _abi.TRI_ERR_INVALID_ARG),
    (dict(mode=7), _abi.TRI_ERR_INVALID_ARG),
    (dict(mode=1, pos=None), _abi.TRI_ERR_INVALID_ARG),
    (dict(K=A + 8), _abi.TRI_ERR_ALIGNMENT),
    (dict(scores=A + 2), _abi.TRI_ERR_ALIGNMENT),
    (dict(c=A + 4), _abi.TRI_ERR_ALIGNMENT),
    (dict(ws=A + 64), _abi.TRI_ERR_ALIGNMENT),
    (dict(ws_bytes=100), _abi.TRI_ERR_WORKSPACE_TOO_SMALL),
    (dict(ws=None), _abi.TRI_ERR_INVALID_ARG),
])
def test_score_rejects_bad_arguments(kwargs, status):
    assert _score(M, _kv(), **kwargs) == status


def test_score_rejects_bad_model_and_layout():
    assert _score(tri.model(1, 32, 8, 1e6, head_dim=96), _kv()) == _abi.TRI_ERR_UNSUPPORTED
    assert _score(tri.model(1, 32, 8, 1e6, head_dim=512), _kv()) == _abi.TRI_ERR_UNSUPPORTED
    assert _score(tri.model(1, 32, 8, 1e6, rope_style=-1), _kv()) == _abi.TRI_ERR_INVALID_ARG
    assert _score(tri.model(1, 30, 8, 1e6), _kv()) == _abi.TRI_ERR_INVALID_ARG
    assert _score(tri.model(1, 32, 8, 0.5), _kv()) == _abi.TRI_ERR_INVALID_ARG
    assert _score(tri.model(0, 32, 8, 1e6), _kv()) == _abi.TRI_ERR_INVALID_ARG
    assert _score(M, None) == _abi.TRI_ERR_INVALID_ARG
    assert _score(M, _kv(layout=5)) == _abi.TRI_ERR_INVALID_ARG
    assert _score(M, _kv(n_seqs=0)) == _abi.TRI_ERR_INVALID_ARG
    assert _score(M, _kv(total=-1)) == _abi.TRI_ERR_INVALID_ARG
    assert _score(M, _kv(row_off=A + 4)) == _abi.TRI_ERR_ALIGNMENT
    # paged: table required, block size must be a power of two
    assert _score(M, _kv(layout=1)) == _abi.TRI_ERR_INVALID_ARG
    assert _score(M, _kv(layout=1, table=A, max_blocks=4, bs=12, nb=8)) == _abi.TRI_ERR_UNSUPPORTED
    assert _score(M, _kv(layout=1, table=A, max_blocks=0, bs=16, nb=8)) == _abi.TRI_ERR_INVALID_ARG


@pytest.mark.parametrize("kwargs,status", [
    (dict(B=0), _abi.TRI_ERR_INVALID_ARG),
    (dict(W=-1), _abi.TRI_ERR_INVALID_ARG),
    (dict(B=8, W=9), _abi.TRI_ERR_INVALID_ARG),
    (dict(Ko=A), _abi.TRI_ERR_INVALID_ARG),          # output aliases the input
    (dict(poso=5 * A, pos=None), _abi.TRI_ERR_INVALID_ARG),
    (dict(V=2 * A + 8), _abi.TRI_ERR_ALIGNMENT),
    (dict(Vo=4 * A + 4), _abi.TRI_ERR_ALIGNMENT),
    (dict(ws_bytes=1024), _abi.TRI_ERR_WORKSPACE_TOO_SMALL),
    (dict(out=_abi.TriOutDesc(1, 0, None, 16, 0, 4)), _abi.TRI_ERR_INVALID_ARG),
    (dict(out=_abi.TriOutDesc(1, 4, A, 24, 0, 4)), _abi.TRI_ERR_UNSUPPORTED),
])
def test_compact_rejects_bad_arguments(kwargs, status):
    assert _compact(M, _kv(), **kwargs) == status


def test_calib_rejects_bad_arguments():
    L = _abi.load()
    assert L.tri_calib(ctypes.byref(M), None, 1024, A, A, None) == _abi.TRI_ERR_INVALID_ARG
    assert L.tri_calib(ctypes.byref(M), A, 0, A, A, None) == _abi.TRI_ERR_INVALID_ARG
    assert L.tri_calib(ctypes.byref(M), A + 2, 8, A, A, None) == _abi.TRI_ERR_ALIGNMENT
    assert L.tri_calib(None, A, 8, A, A, None) == _abi.TRI_ERR_INVALID_ARG


def test_calib_update_rejects_bad_arguments():
    L = _abi.load()

    def upd(q=A, nq=8, decay=0.9, sums=A, w=A, c=A, mn=A, m=M):
        return L.tri_calib_update(ctypes.byref(m) if m is not None else None, q, nq, decay, sums, w, c, mn, None)

    assert upd(q=None) == _abi.TRI_ERR_INVALID_ARG
    assert upd(nq=0) == _abi.TRI_ERR_INVALID_ARG
    assert upd(decay=0.0) == _abi.TRI_ERR_INVALID_ARG
    assert upd(decay=1.5) == _abi.TRI_ERR_INVALID_ARG
    assert upd(decay=float("nan")) == _abi.TRI_ERR_INVALID_ARG
    assert upd(sums=None) == _abi.TRI_ERR_INVALID_ARG
    assert upd(w=None) == _abi.TRI_ERR_INVALID_ARG
    assert upd(sums=A + 4) == _abi.TRI_ERR_ALIGNMENT
    assert upd(q=A + 8) == _abi.TRI_ERR_ALIGNMENT
    assert upd(m=None) == _abi.TRI_ERR_INVALID_ARG
    assert upd(m=tri.model(1, 32, 8, 1e6, head_dim=80)) == _abi.TRI_ERR_UNSUPPORTED


def test_calib_stats_rejects_bad_arguments():
    L = _abi.load()

    def st(n=32, c=A, mn=A, rc=None, rm=None, conc=A, hs=A):
        return L.tri_calib_stats(ctypes.byref(M), n, c, mn, rc, rm, conc, hs, None)

    assert st(n=0) == _abi.TRI_ERR_INVALID_ARG
    assert st(c=None) == _abi.TRI_ERR_INVALID_ARG
    assert st(conc=None, hs=None) == _abi.TRI_ERR_INVALID_ARG
    assert st(rc=A) == _abi.TRI_ERR_INVALID_ARG  # reference centres without reference norms
    assert st(c=A + 4) == _abi.TRI_ERR_ALIGNMENT
    assert st(hs=A + 2) == _abi.TRI_ERR_ALIGNMENT


def test_key_centres_rejects_bad_arguments():
    L = _abi.load()
    need = tri.tri_key_centres_ws_size(M, 1)
    assert need >= 256 + 8 * 16 * 64 * 24 and need % 256 == 0
    assert tri.tri_key_centres_ws_size(M, 0) == 0

    def kc(kv=None, K=A, pos=A, mode=0, c=A, mn=A, ws=A, ws_bytes=1 << 30):
        kv = kv or _kv()
        return L.tri_key_centres(ctypes.byref(M), ctypes.byref(kv), K, pos, mode, c, mn, ws, ws_bytes, None)

    assert kc(K=None) == _abi.TRI_ERR_INVALID_ARG
    assert kc(pos=None) == _abi.TRI_ERR_INVALID_ARG  # a RoPE cache is de-rotated by position
    assert kc(mode=7) == _abi.TRI_ERR_INVALID_ARG
    assert kc(c=None) == _abi.TRI_ERR_INVALID_ARG
    assert kc(K=A + 8) == _abi.TRI_ERR_ALIGNMENT
    assert kc(ws_bytes=need - 1) == _abi.TRI_ERR_WORKSPACE_TOO_SMALL
    assert kc(ws=A + 128) == _abi.TRI_ERR_ALIGNMENT
    assert kc(kv=_kv(layout=1)) == _abi.TRI_ERR_INVALID_ARG


def test_decode_attention_rejects_bad_arguments():
    L = _abi.load()
    need = tri.tri_attention_ws_size(M, 1)
    assert need >= 256 + 8 * 8 * 4 * 130 * 4 and need % 256 == 0

    def at(m=M, kv=None, K=A, V=2 * A, q=3 * A, scale=0.088, out=4 * A, lse=None, ws=5 * A, ws_bytes=1 << 30):
        kv = kv or _kv()
        return L.tri_decode_attention(ctypes.byref(m), ctypes.byref(kv), K, V, q, scale, out, lse, ws, ws_bytes,
                                      None)

    assert at(K=None) == _abi.TRI_ERR_INVALID_ARG
    assert at(V=None) == _abi.TRI_ERR_INVALID_ARG
    assert at(q=None) == _abi.TRI_ERR_INVALID_ARG
    assert at(out=None) == _abi.TRI_ERR_INVALID_ARG
    assert at(scale=0.0) == _abi.TRI_ERR_INVALID_ARG
    assert at(scale=float("inf")) == _abi.TRI_ERR_INVALID_ARG
    assert at(K=A + 8) == _abi.TRI_ERR_ALIGNMENT
    assert at(q=3 * A + 1) == _abi.TRI_ERR_ALIGNMENT
    assert at(lse=A + 2) == _abi.TRI_ERR_ALIGNMENT
    assert at(ws_bytes=need - 1) == _abi.TRI_ERR_WORKSPACE_TOO_SMALL
    assert at(m=tri.model(1, 64, 2, 1e6)) == _abi.TRI_ERR_UNSUPPORTED  # 32 query heads per KV head


def test_score_compact_rejects_bad_arguments():
    L = _abi.load()

    def sc(max_row=4096, scores=None, B=64, W=8, K=A, ws_bytes=1 << 30):
        arr = (ctypes.c_int32 * 3)(1, 2, 4)
        out = _abi.TriOutDesc(0, 0, None, 0, 0, 0)
        return L.tri_score_compact(ctypes.byref(M), ctypes.byref(_kv()), K, 2 * A, None, A, A, A, arr, 3, 0, B, W,
                                   max_row, ctypes.byref(out), 3 * A, 4 * A, None, None, None, scores, A, ws_bytes,
                                   None)

    assert sc(max_row=-1) == _abi.TRI_ERR_INVALID_ARG
    assert sc(max_row=40000) == _abi.TRI_ERR_INVALID_ARG  # the unfused path needs a score buffer
    assert sc(B=0) == _abi.TRI_ERR_INVALID_ARG
    assert sc(W=65) == _abi.TRI_ERR_INVALID_ARG
    assert sc(K=None) == _abi.TRI_ERR_INVALID_ARG
    assert sc(K=A + 8) == _abi.TRI_ERR_ALIGNMENT
    assert sc(ws_bytes=100) == _abi.TRI_ERR_WORKSPACE_TOO_SMALL


def test_status_check_rejects_bad_workspace():
    L = _abi.load()
    assert L.tri_status_check(None, None, None) == _abi.TRI_ERR_INVALID_ARG
    assert L.tri_status_check(A + 16, None, None) == _abi.TRI_ERR_ALIGNMENT


def test_selftest_wait_rejects_bad_arguments():
    """Checked before any launch, so no device is needed."""
    L = _abi.load()
    f = L.tri_selftest_wait_timeout
    assert f(None, 256, 10**6, None) == _abi.TRI_ERR_INVALID_ARG
    assert f(A, 255, 10**6, None) == _abi.TRI_ERR_WORKSPACE_TOO_SMALL
    assert f(A + 16, 256, 10**6, None) == _abi.TRI_ERR_ALIGNMENT
    assert f(A, 256, 999, None) == _abi.TRI_ERR_INVALID_ARG
    assert f(A, 256, 10**10 + 1, None) == _abi.TRI_ERR_INVALID_ARG


def test_header_constants_match_the_binding():
    """Every numeric #define, enum member and status code of include/tri.h has the
    same value in the Python binding, and the binding defines no TRI_ constant the
    header lacks."""
    text = open(os.path.join(ROOT, "include", "tri.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    header = {}
    for name, val in re.findall(r"#define\s+(TRI_[A-Z0-9_]+)\s+(0x[0-9a-fA-F]+|[0-9]+)u?\b", text):
        header[name] = int(val, 0)
    for name, val in re.findall(r"\b(TRI_[A-Z0-9_]+)\s*=\s*(0x[0-9a-fA-F]+|[0-9]+)", text):
        header[name] = int(val, 0)
    assert len(header) >= 20
    binding = {k: v for k, v in vars(_abi).items() if k.startswith("TRI_") and isinstance(v, int)}
    assert header == binding


def test_binding_refuses_pageable_host_records():
    """V and the compacted outputs may be pinned host tensors (the device addresses
    them); pageable host memory is refused before anything is called."""
    t = torch.zeros(64, 128, dtype=torch.bfloat16)
    assert not t.is_pinned()
    with pytest.raises(ValueError, match="pinned"):
        tri._pd(t)
    assert tri._pd(None) is None


def test_binding_refuses_host_and_strided_tensors():
    """A host pointer or a strided view must never reach a kernel."""
    m = tri.model(1, 32, 8, 1e6)
    with pytest.raises(ValueError, match="CUDA tensor"):
        tri.tri_calib(m, torch.zeros(1, 32, 8, 128, dtype=torch.bfloat16), 8, torch.zeros(1, 32, 64, 2),
                      torch.zeros(1, 32, 64))
    with pytest.raises(ValueError, match="CUDA tensor"):
        tri.kv_contig(1, torch.zeros(9, dtype=torch.int64), 0)
