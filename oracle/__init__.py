"""Plain fp64 CPU oracle for TriAttention key scoring, selection and compaction.

TEST INFRASTRUCTURE ONLY.  The test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers allowed; the product path
(``kv_cache_compression_calib_b200``) never imports this package, and this
package never imports it.  The arithmetic lives in ``tri_oracle.c`` (built to
``libtri_oracle.so`` by :func:`build`); this module only marshals numpy arrays.

Sources of what is computed: "TriAttention：基于三角函数 KV 压缩的高效长推理"
(whatsmy.fun paper digest), section 流程详解 steps 1-4, and the
"WeianMao/triattention" project card, section "How it works".  The exact rule
is written out in the header of ``tri_oracle.c``.

Parity pins for every function here are in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tri_oracle.c")
_LIB = os.path.join(_HERE, "libtri_oracle.so")
_lib = None

_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile ``tri_oracle.c`` into ``libtri_oracle.so`` (gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def load(path: str):
    """Load a build of ``tri_oracle.c`` from ``path`` and declare its signatures."""
    L = ctypes.CDLL(path)
    _declare(L)
    return L


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = load(_LIB)
    return _lib


def _declare(L) -> None:
    L.ora_omega.restype = ctypes.c_double
    L.ora_omega.argtypes = [ctypes.c_double, ctypes.c_int, ctypes.c_int]
    L.ora_num_threads.restype = ctypes.c_int
    L.ora_num_threads.argtypes = []
    L.ora_trig_series.restype = ctypes.c_double
    L.ora_trig_series.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double, _f64p, _f64p, ctypes.c_int64]
    L.ora_calib.restype = None
    L.ora_calib.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int64, _f64p, _f64p, _f64p]
    score_args = [ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int, _f64p, _f64p, ctypes.c_int64,
                  _f64p, _i64p, ctypes.c_int, ctypes.c_int64, ctypes.c_int, _i64p, _f64p]
    for name in ("ora_score_literal", "ora_score_collapsed", "ora_score_absorbed"):
        fn = getattr(L, name)
        fn.restype = None
        fn.argtypes = score_args
    L.ora_calib_online.restype = None
    L.ora_calib_online.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int64, _f64p, _i64p, ctypes.c_int64,
                                   ctypes.c_double, _f64p, _f64p]
    L.ora_key_centres.restype = None
    L.ora_key_centres.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int64, _f64p, _i64p,
                                  ctypes.c_int, _f64p, _f64p]
    L.ora_calib_stats.restype = None
    L.ora_calib_stats.argtypes = [ctypes.c_int, _f64p, _f64p, ctypes.c_void_p, ctypes.c_void_p, _f64p, _f64p]
    L.ora_attention.restype = None
    L.ora_attention.argtypes = [ctypes.c_int, ctypes.c_int64, _f64p, _f64p, _f64p, ctypes.c_double, _f64p,
                                ctypes.POINTER(ctypes.c_double)]
    L.ora_select.restype = ctypes.c_int64
    L.ora_select.argtypes = [ctypes.c_int64, _f64p, ctypes.c_int64, ctypes.c_int64, _i64p]
    L.ora_gather_bytes.restype = None
    L.ora_gather_bytes.argtypes = [ctypes.c_int64, _i64p, ctypes.c_int64, _u8p, _u8p]


def num_threads() -> int:
    return int(lib().ora_num_threads())


# ----------------------------------------------------------------- helpers

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bit patterns (uint16 / int16) exactly to float64."""
    u = np.ascontiguousarray(bits).view(np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def e4m3_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of OCP fp8 e4m3 ("fn") codes: sign, 4 exponent bits (bias 7),
    3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6); no infinities, and the
    codes 0x7f / 0xff are NaN."""
    b = np.ascontiguousarray(bits).view(np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    out = sign * mag
    out[(b & 0x7F) == 0x7F] = np.nan
    return out


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _i64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int64)


def omega(theta: float, d: int) -> np.ndarray:
    """w_f = theta^(-2f/d) for f < d/2."""
    return np.array([lib().ora_omega(theta, d, f) for f in range(d // 2)])


def trig_series(theta: float, qbar: np.ndarray, k_pre: np.ndarray, dist: int,
                interleaved: bool = False) -> float:
    """sum_f |qbar_f||k_f| cos(w_f dist + arg qbar_f - arg k_f); qbar [F][2], k_pre [d].

    Pair f is dims (f, f+d/2) (rotate-half), or (2f, 2f+1) when ``interleaved``."""
    k_pre = _f64(k_pre)
    return float(lib().ora_trig_series(k_pre.shape[0], int(bool(interleaved)), theta, _f64(qbar), k_pre,
                                       int(dist)))


def calib(q: np.ndarray, interleaved: bool = False):
    """Per-pair complex centre and mean magnitude of pre-RoPE queries q [nq][d].

    Returns (centre [F][2], mnorm [F])."""
    q = _f64(q)
    nq, d = q.shape
    centre = np.empty((d // 2, 2))
    mnorm = np.empty(d // 2)
    lib().ora_calib(d, int(bool(interleaved)), nq, q, centre, mnorm)
    return centre, mnorm


def calib_online(batches, decay: float = 1.0, interleaved: bool = False):
    """Centres after a stream of query batches (each [n_b][d]) where every new batch
    multiplies the weight of all earlier queries by ``decay``.  Returns (centre, mnorm)."""
    q = _f64(np.concatenate([np.asarray(b, dtype=np.float64) for b in batches], axis=0))
    upd = _i64(np.concatenate([np.full(len(b), i) for i, b in enumerate(batches)]))
    d = q.shape[1]
    centre = np.empty((d // 2, 2))
    mnorm = np.empty(d // 2)
    lib().ora_calib_online(d, int(bool(interleaved)), q.shape[0], q, upd, len(batches), float(decay), centre,
                           mnorm)
    return centre, mnorm


def key_centres(theta: float, keys: np.ndarray, pos: np.ndarray, post_rope: bool,
                interleaved: bool = False):
    """Pre-RoPE key centre [F][2] and mean magnitude [F] of one row's keys [n][d]
    (de-rotated by their positions when ``post_rope``)."""
    keys = _f64(keys)
    n, d = keys.shape
    pos = _i64(pos)
    centre = np.empty((d // 2, 2))
    mnorm = np.empty(d // 2)
    lib().ora_key_centres(d, int(bool(interleaved)), float(theta), n, keys, pos, 1 if post_rope else 0, centre,
                          mnorm)
    return centre, mnorm


def calib_stats(centre: np.ndarray, mnorm: np.ndarray, ref_centre=None, ref_mnorm=None):
    """(concentration [F], (head concentration, drift vs the reference)) of one head."""
    centre = _f64(centre)
    mnorm = _f64(mnorm)
    F = mnorm.shape[0]
    conc = np.empty(F)
    head = np.empty(2)
    if ref_centre is None:
        lib().ora_calib_stats(F, centre, mnorm, None, None, conc, head)
    else:
        rc, rm = _f64(ref_centre), _f64(ref_mnorm)
        lib().ora_calib_stats(F, centre, mnorm, rc.ctypes.data_as(ctypes.c_void_p),
                              rm.ctypes.data_as(ctypes.c_void_p), conc, head)
    return conc, (float(head[0]), float(head[1]))


def attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float):
    """Softmax attention of one query [d] over keys/values [n][d]: (out [d], lse)."""
    q = _f64(q)
    keys = _f64(keys).reshape(-1, q.shape[0])
    values = _f64(values).reshape(-1, q.shape[0])
    out = np.empty(q.shape[0])
    lse = ctypes.c_double(0.0)
    lib().ora_attention(q.shape[0], keys.shape[0], q, keys, values, float(scale), out, ctypes.byref(lse))
    return out, float(lse.value)


def _score(fn, theta, qbar, mnorm, keys, pos, post_rope, p_now, offsets, interleaved=False):
    qbar = _f64(qbar)
    mnorm = _f64(mnorm)
    keys = _f64(keys)
    n, d = keys.shape
    G = qbar.shape[0]
    assert qbar.shape == (G, d // 2, 2) and mnorm.shape == (G, d // 2)
    pos = _i64(pos)
    assert pos.shape == (n,)
    offs = _i64(offsets)
    out = np.empty(n)
    fn(d, int(bool(interleaved)), float(theta), G, qbar, mnorm, n, keys, pos, 1 if post_rope else 0,
       int(p_now), offs.shape[0], offs, out)
    return out


def score_literal(theta, qbar, mnorm, keys, pos, post_rope, p_now, offsets,
                  interleaved=False) -> np.ndarray:
    """Literal triple sum (g, f, delta).  qbar [G][F][2], mnorm [G][F], keys [n][d]."""
    return _score(lib().ora_score_literal, theta, qbar, mnorm, keys, pos, post_rope, p_now, offsets,
                  interleaved)


def score_collapsed(theta, qbar, mnorm, keys, pos, post_rope, p_now, offsets,
                    interleaved=False) -> np.ndarray:
    """Delta sum folded by angle addition: one (cos, sin) per (key, g, f)."""
    return _score(lib().ora_score_collapsed, theta, qbar, mnorm, keys, pos, post_rope, p_now,
                  offsets, interleaved)


def score_absorbed(theta, qbar, mnorm, keys, pos, post_rope, p_now, offsets,
                   interleaved=False) -> np.ndarray:
    """Linear form sum_f Re(A_f conj k_f) + c_f |k_f| (identity cross-check only)."""
    return _score(lib().ora_score_absorbed, theta, qbar, mnorm, keys, pos, post_rope, p_now,
                  offsets, interleaved)


def select(score: np.ndarray, B: int, W: int) -> np.ndarray:
    """Ascending kept slots of one row: last W slots + best (B-W) of the rest."""
    score = _f64(score)
    n = score.shape[0]
    kept = np.empty(max(n, 1), dtype=np.int64)  # room for n so a faulty count cannot overrun
    c = lib().ora_select(n, score, int(B), int(W), kept)
    if c < 0:
        raise ValueError(f"invalid selection arguments B={B} W={W}")
    return kept[:c]


def gather(src: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Stable gather of rows of ``src`` (any dtype) by ``idx``: out[t] = src[idx[t]]."""
    src = np.ascontiguousarray(src)
    idx = _i64(idx)
    width = src.dtype.itemsize * (int(np.prod(src.shape[1:])) if src.ndim > 1 else 1)
    out = np.empty((idx.shape[0],) + src.shape[1:], dtype=src.dtype)
    if idx.size:
        assert idx.min() >= 0 and idx.max() < src.shape[0]
        lib().ora_gather_bytes(idx.shape[0], idx, width, src.view(np.uint8).reshape(-1),
                               out.view(np.uint8).reshape(-1))
    return out


def row_scores(theta, centres, mnorms, h, G, keys, pos, post_rope, p_now, offsets,
               tier: str = "collapsed", interleaved: bool = False) -> np.ndarray:
    """Scores of one cache row of KV head ``h``: query heads h*G .. h*G+G-1 of one layer.

    centres [Hq][F][2], mnorms [Hq][F] (one layer); keys [n][d] float64.
    The query heads of KV head h are taken as the contiguous group
    [h*G, (h+1)*G) (the grouped-query layout of Qwen3-style models)."""
    qb = _f64(centres)[h * G:(h + 1) * G]
    mn = _f64(mnorms)[h * G:(h + 1) * G]
    fn = {"literal": score_literal, "collapsed": score_collapsed, "absorbed": score_absorbed}[tier]
    return fn(theta, qb, mn, keys, pos, post_rope, p_now, offsets, interleaved)
