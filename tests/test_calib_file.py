"""Calibration files (tri_calib_save / tri_calib_load): the offline centres of
"TriAttention：基于三角函数 KV 压缩的高效长推理" (流程详解 step 1) stored with the
model shape and query count they came from (复现注意事项: the centres depend on
the calibration data).  Host-side file I/O only, so these run without a GPU.

The byte layout is pinned by building the expected file independently with
`struct` (little-endian header, FNV-1a 64-bit payload hash written out from its
definition) and comparing bytes; loads must reproduce every stored bit (NaN
payloads, -0.0, subnormals included) and refuse damaged files."""
import ctypes
import os
import struct

import numpy as np
import pytest
import torch

import kv_cache_compression_calib_b200 as tri
from kv_cache_compression_calib_b200 import _abi


def fnv1a64(data: bytes) -> int:
    h = 0xcbf29ce484222325
    for b in data:
        h ^= b
        h = (h * 0x100000001b3) & 0xFFFFFFFFFFFFFFFF
    return h


def expected_file(m, nq, c, n) -> bytes:
    payload = np.ascontiguousarray(c, dtype="<f4").tobytes() + np.ascontiguousarray(n, dtype="<f4").tobytes()
    hdr = b"TRICALIB" + struct.pack("<IIiiiiiidqQ", 1, 64, m.head_dim, m.n_layers, m.n_q_heads, m.n_kv_heads,
                                    m.rope_style, 0, m.rope_theta, nq, fnv1a64(payload))
    assert len(hdr) == 64
    return hdr + payload


def special_centres(m, seed=3):
    rng = np.random.default_rng(seed)
    F = m.head_dim // 2
    c = rng.standard_normal((m.n_layers, m.n_q_heads, F, 2)).astype(np.float32)
    n = np.abs(rng.standard_normal((m.n_layers, m.n_q_heads, F))).astype(np.float32)
    flat = c.reshape(-1)
    flat[0] = -0.0
    flat[1] = np.float32(1e-42)  # subnormal
    flat[2:3].view(np.uint32)[0] = 0x7FC01234  # NaN with a payload
    flat[3] = np.inf
    return c, n


@pytest.mark.parametrize("d,style", [(128, tri.TRI_ROPE_HALF), (64, tri.TRI_ROPE_INTERLEAVED),
                                     (256, tri.TRI_ROPE_HALF)])
def test_save_writes_the_documented_bytes_and_load_returns_every_bit(tmp_path, d, style):
    m = tri.model(3, 8, 2, 1e6 if d == 128 else 1e4, head_dim=d, rope_style=style)
    c, n = special_centres(m)
    path = tmp_path / "calib.tri"
    tri.tri_calib_save(path, m, 1024, torch.from_numpy(c), torch.from_numpy(n))
    assert path.read_bytes() == expected_file(m, 1024, c, n)
    m2, nq, c2, n2 = tri.tri_calib_load(path)
    assert (m2.head_dim, m2.n_layers, m2.n_q_heads, m2.n_kv_heads, m2.rope_theta, m2.rope_style) == \
        (m.head_dim, m.n_layers, m.n_q_heads, m.n_kv_heads, m.rope_theta, m.rope_style)
    assert nq == 1024
    assert np.array_equal(c2.numpy().view(np.uint32), c.view(np.uint32))
    assert np.array_equal(n2.numpy().view(np.uint32), n.view(np.uint32))


def _load_raw(path, cap):
    L = _abi.load()
    m = _abi.TriModel()
    nq = ctypes.c_int64(-1)
    c = np.full(cap * 2, 7.0, dtype=np.float32)
    n = np.full(cap, 7.0, dtype=np.float32)
    st = L.tri_calib_load(str(path).encode(), ctypes.byref(m), ctypes.byref(nq), c.ctypes.data, n.ctypes.data, cap)
    return st, m, nq.value, c, n


def test_load_refuses_damaged_files(tmp_path):
    m = tri.model(2, 4, 4, 1e6)
    c, n = special_centres(m)
    good = expected_file(m, 64, c, n)
    pairs = 2 * 4 * 64
    cases = {
        "magic": b"TRICALIX" + good[8:],
        "version": good[:8] + struct.pack("<I", 2) + good[12:],
        "header size": good[:12] + struct.pack("<I", 72) + good[16:],
        "head dim": good[:16] + struct.pack("<i", 96) + good[20:],
        "heads": good[:24] + struct.pack("<ii", 4, 3) + good[32:],
        "rope style": good[:32] + struct.pack("<i", 5) + good[36:],
        "reserved": good[:36] + struct.pack("<i", 1) + good[40:],
        "theta": good[:40] + struct.pack("<d", 0.5) + good[48:],
        "nq": good[:48] + struct.pack("<q", 0) + good[56:],
        "hash": good[:56] + struct.pack("<Q", fnv1a64(good[64:]) ^ 1) + good[64:],
        "payload bit": good[:100] + bytes([good[100] ^ 0x10]) + good[101:],
        "truncated": good[:-4],
        "trailing": good + b"\0",
        "header only": good[:64],
        "empty": b"",
    }
    for name, data in cases.items():
        p = tmp_path / f"bad_{name.replace(' ', '_')}.tri"
        p.write_bytes(data)
        st, _, nq, cbuf, nbuf = _load_raw(p, pairs)
        assert st == _abi.TRI_ERR_IO, name
        assert nq == -1 and np.all(cbuf == 7.0) and np.all(nbuf == 7.0), name  # outputs untouched
    st, *_ = _load_raw(tmp_path / "missing.tri", pairs)
    assert st == _abi.TRI_ERR_IO


def test_load_checks_capacity_and_header_only_reads(tmp_path):
    m = tri.model(2, 4, 4, 1e6)
    c, n = special_centres(m)
    p = tmp_path / "c.tri"
    p.write_bytes(expected_file(m, 5, c, n))
    pairs = 2 * 4 * 64
    st, *_ = _load_raw(p, pairs - 1)
    assert st == _abi.TRI_ERR_WORKSPACE_TOO_SMALL
    L = _abi.load()
    m2 = _abi.TriModel()
    nq = ctypes.c_int64(0)
    assert L.tri_calib_load(str(p).encode(), ctypes.byref(m2), ctypes.byref(nq), None, None, 0) == 0
    assert (m2.n_layers, m2.n_q_heads, m2.head_dim, nq.value) == (2, 4, 128, 5)
    # one output NULL and the other not is an argument error
    cbuf = np.zeros(pairs * 2, dtype=np.float32)
    assert L.tri_calib_load(str(p).encode(), ctypes.byref(m2), ctypes.byref(nq), cbuf.ctypes.data, None,
                            pairs) == _abi.TRI_ERR_INVALID_ARG


def test_save_rejects_bad_arguments(tmp_path):
    L = _abi.load()
    m = tri.model(1, 4, 4, 1e6)
    buf = np.zeros(4 * 64 * 2, dtype=np.float32)
    p = str(tmp_path / "x.tri").encode()
    assert L.tri_calib_save(None, ctypes.byref(m), 1, buf.ctypes.data, buf.ctypes.data) == _abi.TRI_ERR_INVALID_ARG
    assert L.tri_calib_save(p, ctypes.byref(m), 0, buf.ctypes.data, buf.ctypes.data) == _abi.TRI_ERR_INVALID_ARG
    assert L.tri_calib_save(p, ctypes.byref(m), 1, None, buf.ctypes.data) == _abi.TRI_ERR_INVALID_ARG
    bad = tri.model(1, 4, 3, 1e6)  # 4 query heads over 3 KV heads
    assert L.tri_calib_save(p, ctypes.byref(bad), 1, buf.ctypes.data, buf.ctypes.data) == _abi.TRI_ERR_INVALID_ARG
    unwritable = str(tmp_path / "no_such_dir" / "x.tri").encode()
    assert L.tri_calib_save(unwritable, ctypes.byref(m), 1, buf.ctypes.data, buf.ctypes.data) == _abi.TRI_ERR_IO
    assert not os.path.exists(tmp_path / "x.tri")
