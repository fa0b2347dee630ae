"""ctypes declarations of libtri.so (mirrors include/tri.h)."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtri.so")

TRI_OK = 0
TRI_ERR_INVALID_ARG = 1
TRI_ERR_UNSUPPORTED = 2
TRI_ERR_ALIGNMENT = 3
TRI_ERR_WORKSPACE_TOO_SMALL = 4
TRI_ERR_CUDA = 5
TRI_ERR_DEVICE_FLAG = 6
TRI_ERR_IO = 7

TRI_FLAG_ROW_OFFSETS = 0x1
TRI_FLAG_NONFINITE = 0x2
TRI_FLAG_BLOCK_TABLE = 0x4
TRI_FLAG_STAGE_TIMEOUT = 0x8

TRI_MAX_OFFSETS = 64
TRI_ROPE_HALF = 0
TRI_ROPE_INTERLEAVED = 1
TRI_KV_CONTIG = 0
TRI_KV_PAGED = 1
TRI_ELEM_BF16 = 0
TRI_ELEM_FP8_E4M3 = 1
TRI_KEYS_POST_ROPE = 0
TRI_KEYS_PRE_ROPE = 1

# Every symbol include/tri.h declares.
EXPORTS = ("tri_status_str", "tri_version", "tri_last_error", "tri_workspace_size", "tri_workspace_init", "tri_calib",
           "tri_score", "tri_compact", "tri_status_check", "tri_score_noalloc", "tri_calib_update",
           "tri_calib_stats", "tri_key_centres_ws_size", "tri_key_centres", "tri_attention_ws_size",
           "tri_decode_attention", "tri_score_compact", "tri_selftest_wait_timeout", "tri_calib_save",
           "tri_calib_load", "tri_decode_attention_tc")
TRI_FUSED_MAX_ROW = 32768
TRI_FUSED_PREFER_ROW = 8192
TRI_NOALLOC_MAX_ROWS = 4096
TRI_CALIB_FILE_VERSION = 1


class TriModel(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int32), ("n_layers", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("rope_theta", ctypes.c_double), ("rope_style", ctypes.c_int32),
                ("pad_", ctypes.c_int32)]


class TriKvDesc(ctypes.Structure):
    _fields_ = [("layout", ctypes.c_int32), ("n_seqs", ctypes.c_int32),
                ("total_keys", ctypes.c_int64), ("row_off", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("max_blocks", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("n_blocks", ctypes.c_int64),
                ("elem_type", ctypes.c_int32), ("pad_", ctypes.c_int32)]


class TriOutDesc(ctypes.Structure):
    _fields_ = [("layout", ctypes.c_int32), ("max_blocks", ctypes.c_int32),
                ("block_table", ctypes.c_void_p), ("block_size", ctypes.c_int32),
                ("pad_", ctypes.c_int32), ("n_blocks", ctypes.c_int64)]


_P = ctypes.c_void_p
_lib = None


def load(path: str = LIB_PATH):
    """Load libtri.so and declare every entry point.  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libtri.so not built at {path}: run kv_cache_compression_calib_b200/build.py")
    L = ctypes.CDLL(path)
    L.tri_status_str.restype = ctypes.c_char_p
    L.tri_status_str.argtypes = [ctypes.c_int]
    L.tri_version.restype = ctypes.c_uint32
    L.tri_version.argtypes = []
    L.tri_last_error.restype = ctypes.c_char_p
    L.tri_last_error.argtypes = []
    L.tri_workspace_size.restype = ctypes.c_size_t
    L.tri_workspace_size.argtypes = [ctypes.POINTER(TriModel), ctypes.c_int32, ctypes.c_int32]
    L.tri_workspace_init.restype = ctypes.c_int
    L.tri_workspace_init.argtypes = [_P, ctypes.c_size_t, _P]
    L.tri_calib.restype = ctypes.c_int
    L.tri_calib.argtypes = [ctypes.POINTER(TriModel), _P, ctypes.c_int64, _P, _P, _P]
    L.tri_calib_update.restype = ctypes.c_int
    L.tri_calib_update.argtypes = [ctypes.POINTER(TriModel), _P, ctypes.c_int64, ctypes.c_double, _P, _P, _P, _P,
                                   _P]
    L.tri_calib_stats.restype = ctypes.c_int
    L.tri_calib_stats.argtypes = [ctypes.POINTER(TriModel), ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P]
    L.tri_score_compact.restype = ctypes.c_int
    L.tri_score_compact.argtypes = [ctypes.POINTER(TriModel), ctypes.POINTER(TriKvDesc), _P, _P, _P, _P, _P, _P, _P,
                                    ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                    ctypes.POINTER(TriOutDesc), _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
    L.tri_attention_ws_size.restype = ctypes.c_size_t
    L.tri_attention_ws_size.argtypes = [ctypes.POINTER(TriModel), ctypes.c_int32]
    L.tri_decode_attention.restype = ctypes.c_int
    L.tri_decode_attention.argtypes = [ctypes.POINTER(TriModel), ctypes.POINTER(TriKvDesc), _P, _P, _P,
                                       ctypes.c_float, _P, _P, _P, ctypes.c_size_t, _P]
    L.tri_decode_attention_tc.restype = ctypes.c_int
    L.tri_decode_attention_tc.argtypes = L.tri_decode_attention.argtypes
    L.tri_key_centres_ws_size.restype = ctypes.c_size_t
    L.tri_key_centres_ws_size.argtypes = [ctypes.POINTER(TriModel), ctypes.c_int32]
    L.tri_key_centres.restype = ctypes.c_int
    L.tri_key_centres.argtypes = [ctypes.POINTER(TriModel), ctypes.POINTER(TriKvDesc), _P, _P, ctypes.c_int32, _P,
                                  _P, _P, ctypes.c_size_t, _P]
    L.tri_score.restype = ctypes.c_int
    L.tri_score.argtypes = [ctypes.POINTER(TriModel), ctypes.POINTER(TriKvDesc), _P, _P, _P, _P, _P,
                            ctypes.POINTER(ctypes.c_int32), ctypes.c_int32, ctypes.c_int32, _P, _P,
                            ctypes.c_size_t, _P]
    L.tri_compact.restype = ctypes.c_int
    L.tri_compact.argtypes = [ctypes.POINTER(TriModel), ctypes.POINTER(TriKvDesc), _P, ctypes.c_int32,
                              ctypes.c_int32, _P, _P, _P, ctypes.POINTER(TriOutDesc), _P, _P, _P, _P,
                              _P, _P, ctypes.c_size_t, _P]
    L.tri_status_check.restype = ctypes.c_int
    L.tri_status_check.argtypes = [_P, ctypes.POINTER(ctypes.c_uint32), _P]
    L.tri_calib_save.restype = ctypes.c_int
    L.tri_calib_save.argtypes = [ctypes.c_char_p, ctypes.POINTER(TriModel), ctypes.c_int64, _P, _P]
    L.tri_calib_load.restype = ctypes.c_int
    L.tri_calib_load.argtypes = [ctypes.c_char_p, ctypes.POINTER(TriModel), ctypes.POINTER(ctypes.c_int64), _P, _P,
                                 ctypes.c_size_t]
    L.tri_selftest_wait_timeout.restype = ctypes.c_int
    L.tri_selftest_wait_timeout.argtypes = [_P, ctypes.c_size_t, ctypes.c_uint64, _P]
    L.tri_score_noalloc.restype = ctypes.c_int
    L.tri_score_noalloc.argtypes = [ctypes.POINTER(TriModel), ctypes.POINTER(TriKvDesc), _P, _P, _P, _P,
                                    _P, ctypes.POINTER(ctypes.c_int32), ctypes.c_int32, ctypes.c_int32,
                                    _P, _P]
    _lib = L
    return L
