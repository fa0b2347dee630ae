"""B200-native TriAttention KV-cache key scoring, top-B selection and compaction.

A thin binding over ``libtri.so`` (C ABI in ``include/tri.h``): the functions
below only marshal torch tensors into pointers and sizes; every step of the
computation runs in the library's sm_100a CUDA kernels.  Importing the package
fails if the library has not been built (``build.py``) - there is no other
implementation to fall back to.

Method: "TriAttention：基于三角函数 KV 压缩的高效长推理" (whatsmy.fun paper
digest), section 流程详解 steps 1-4 - calibrate pre-RoPE query centres, score
each cached key by a trigonometric series in its RoPE distance plus a norm
term, keep the top keys per KV head, compact the cache.
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi
from ._abi import (TRI_ELEM_BF16, TRI_ELEM_FP8_E4M3, TRI_FLAG_BLOCK_TABLE,  # noqa: F401
                   TRI_FLAG_NONFINITE, TRI_FLAG_ROW_OFFSETS, TRI_FLAG_STAGE_TIMEOUT,
                   TRI_KEYS_POST_ROPE, TRI_KEYS_PRE_ROPE, TRI_KV_CONTIG, TRI_KV_PAGED,
                   TRI_MAX_OFFSETS, TRI_ROPE_HALF, TRI_ROPE_INTERLEAVED, TriKvDesc, TriModel, TriOutDesc)

_L = _abi.load()


class TriError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {_L.tri_status_str(status).decode()}"
        if status == _abi.TRI_ERR_CUDA:
            msg += f" [{_L.tri_last_error().decode()}]"
        super().__init__(msg)


def _check(st: int, what: str) -> None:
    if st != _abi.TRI_OK:
        raise TriError(st, what)


def _p(t):
    """Device pointer of a tensor argument (None -> NULL).  Every tensor the library
    reads or writes must be a contiguous CUDA tensor: a host pointer handed to a
    kernel would fault, a strided view would be read as if it were dense."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"expected a CUDA tensor, got one on {t.device}")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor (call .contiguous())")
    return ctypes.c_void_p(t.data_ptr())


def _pd(t):
    """Pointer of a tensor the gather reads or writes record by record (V and the
    compacted outputs): a contiguous CUDA tensor, or a contiguous page-locked host
    tensor, which the device addresses at the same pointer under unified
    addressing - the kept records then cross the host link directly.  Pageable
    host memory is refused: the device cannot address it."""
    if t is not None and not t.is_cuda:
        if not t.is_pinned():
            raise ValueError("expected a CUDA tensor or a pinned (page-locked) host tensor")
        if not t.is_contiguous():
            raise ValueError("expected a contiguous tensor (call .contiguous())")
        return ctypes.c_void_p(t.data_ptr())
    return _p(t)


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def version() -> int:
    return int(_L.tri_version())


def library_path() -> str:
    return _abi.LIB_PATH


# ------------------------------------------------------------- descriptors

def model(n_layers: int, n_q_heads: int, n_kv_heads: int, rope_theta: float,
          head_dim: int = 128, rope_style: int = TRI_ROPE_HALF) -> TriModel:
    """Model shape; ``rope_style`` TRI_ROPE_HALF pairs dims (f, f+d/2), TRI_ROPE_INTERLEAVED (2f, 2f+1)."""
    return TriModel(head_dim, n_layers, n_q_heads, n_kv_heads, float(rope_theta), int(rope_style), 0)


# A descriptor holds raw device pointers; it also keeps a reference to the tensors
# they point into, so the memory cannot be freed (and reused) while it is alive.

def elem_type_of(t: torch.Tensor) -> int:
    """TRI_ELEM_* of a K/V tensor (bf16 or float8_e4m3fn)."""
    if t.dtype == torch.bfloat16:
        return TRI_ELEM_BF16
    if t.dtype == torch.float8_e4m3fn:
        return TRI_ELEM_FP8_E4M3
    raise TypeError(f"unsupported K/V dtype {t.dtype}")


def kv_contig(n_seqs: int, row_off: torch.Tensor, total_keys: int,
              elem_type: int = TRI_ELEM_BF16) -> TriKvDesc:
    """Rows laid end to end; ``row_off`` int64 [R+1] on the device."""
    d = TriKvDesc(TRI_KV_CONTIG, n_seqs, int(total_keys), _p(row_off).value, None, 0, 0, 0,
                  int(elem_type), 0)
    d._keep = (row_off,)
    return d


def kv_paged(n_seqs: int, row_off: torch.Tensor, total_keys: int, block_table: torch.Tensor,
             block_size: int, n_blocks: int, elem_type: int = TRI_ELEM_BF16) -> TriKvDesc:
    """vLLM block layout; ``block_table`` int32 [S][max_blocks] on the device."""
    d = TriKvDesc(TRI_KV_PAGED, n_seqs, int(total_keys), _p(row_off).value,
                  _p(block_table).value, block_table.shape[1], block_size, int(n_blocks),
                  int(elem_type), 0)
    d._keep = (row_off, block_table)
    return d


def out_contig() -> TriOutDesc:
    return TriOutDesc(TRI_KV_CONTIG, 0, None, 0, 0, 0)


def out_paged(block_table: torch.Tensor, block_size: int, n_blocks: int) -> TriOutDesc:
    d = TriOutDesc(TRI_KV_PAGED, block_table.shape[1], _p(block_table).value, block_size, 0,
                   int(n_blocks))
    d._keep = (block_table,)
    return d


# ------------------------------------------------------------------- calls

def tri_workspace_size(m: TriModel, n_seqs: int, B: int) -> int:
    return int(_L.tri_workspace_size(ctypes.byref(m), n_seqs, B))


def tri_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check(_L.tri_workspace_init(_p(ws), ws.numel() * ws.element_size(), _s(stream)),
           "tri_workspace_init")


def alloc_workspace(m: TriModel, n_seqs: int, B: int, device=None, stream=None) -> torch.Tensor:
    """Allocate (through torch) and initialise a workspace for ``tri_score``/``tri_compact``."""
    n = tri_workspace_size(m, n_seqs, B)
    if n == 0:
        raise TriError(_abi.TRI_ERR_INVALID_ARG, "tri_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    tri_workspace_init(ws, stream)
    return ws


def tri_calib(m: TriModel, qpre: torch.Tensor, nq: int, centres: torch.Tensor,
              mean_norm: torch.Tensor, stream=None) -> None:
    _check(_L.tri_calib(ctypes.byref(m), _p(qpre), int(nq), _p(centres), _p(mean_norm), _s(stream)),
           "tri_calib")


def tri_score(m: TriModel, kv: TriKvDesc, K: torch.Tensor, pos, centres: torch.Tensor,
              mean_norm: torch.Tensor, p_now: torch.Tensor, offsets, key_mode: int,
              scores: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    offs = (ctypes.c_int32 * max(len(offsets), 1))(*[int(o) for o in offsets])
    _check(_L.tri_score(ctypes.byref(m), ctypes.byref(kv), _p(K), _p(pos), _p(centres),
                        _p(mean_norm), _p(p_now), offs, len(offsets), int(key_mode), _p(scores),
                        _p(ws), ws.numel() * ws.element_size(), _s(stream)), "tri_score")


def tri_compact(m: TriModel, kv: TriKvDesc, scores: torch.Tensor, B: int, W: int,
                K: torch.Tensor, V: torch.Tensor, pos, out: TriOutDesc, K_out: torch.Tensor,
                V_out: torch.Tensor, pos_out, kept_idx, kept_count, ws: torch.Tensor,
                stream=None) -> None:
    _check(_L.tri_compact(ctypes.byref(m), ctypes.byref(kv), _p(scores), int(B), int(W), _p(K),
                          _pd(V), _p(pos), ctypes.byref(out), _pd(K_out), _pd(V_out), _pd(pos_out),
                          _p(kept_idx), _p(kept_count), _p(ws), ws.numel() * ws.element_size(),
                          _s(stream)), "tri_compact")


def tri_calib_update(m: TriModel, qpre: torch.Tensor, nq: int, decay: float, sums: torch.Tensor,
                     weight: torch.Tensor, centres: torch.Tensor, mean_norm: torch.Tensor, stream=None) -> None:
    """Fold a batch of pre-RoPE queries into the decayed running statistics (fp64
    ``sums`` [L][Hq][d/2][3], ``weight`` [L][Hq]) and write the updated centres."""
    _check(_L.tri_calib_update(ctypes.byref(m), _p(qpre), int(nq), float(decay), _p(sums), _p(weight), _p(centres),
                               _p(mean_norm), _s(stream)), "tri_calib_update")


def tri_calib_stats(m: TriModel, n_heads: int, centres: torch.Tensor, mean_norm: torch.Tensor,
                    ref_centres=None, ref_mean_norm=None, concentration=None, head_stats=None,
                    stream=None) -> None:
    """Per-pair concentration and per-head (concentration, drift vs the reference)."""
    _check(_L.tri_calib_stats(ctypes.byref(m), int(n_heads), _p(centres), _p(mean_norm), _p(ref_centres),
                              _p(ref_mean_norm), _p(concentration), _p(head_stats), _s(stream)),
           "tri_calib_stats")


def tri_key_centres_ws_size(m: TriModel, n_seqs: int) -> int:
    return int(_L.tri_key_centres_ws_size(ctypes.byref(m), int(n_seqs)))


def tri_key_centres(m: TriModel, kv: TriKvDesc, K: torch.Tensor, pos, key_mode: int, centres: torch.Tensor,
                    mean_norm: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    """Pre-RoPE key centre [R][d/2][2] and mean magnitude [R][d/2] of every cache row."""
    _check(_L.tri_key_centres(ctypes.byref(m), ctypes.byref(kv), _p(K), _p(pos), int(key_mode), _p(centres),
                              _p(mean_norm), _p(ws), ws.numel() * ws.element_size(), _s(stream)),
           "tri_key_centres")


def alloc_key_centres_workspace(m: TriModel, n_seqs: int, device=None, stream=None) -> torch.Tensor:
    n = tri_key_centres_ws_size(m, n_seqs)
    if n == 0:
        raise TriError(_abi.TRI_ERR_INVALID_ARG, "tri_key_centres_ws_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    tri_workspace_init(ws, stream)
    return ws


def tri_attention_ws_size(m: TriModel, n_seqs: int) -> int:
    return int(_L.tri_attention_ws_size(ctypes.byref(m), int(n_seqs)))


def alloc_attention_workspace(m: TriModel, n_seqs: int, device=None, stream=None) -> torch.Tensor:
    n = tri_attention_ws_size(m, n_seqs)
    if n == 0:
        raise TriError(_abi.TRI_ERR_INVALID_ARG, "tri_attention_ws_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    tri_workspace_init(ws, stream)
    return ws


def tri_decode_attention(m: TriModel, kv: TriKvDesc, K: torch.Tensor, V: torch.Tensor, q: torch.Tensor,
                         softmax_scale: float, out: torch.Tensor, lse, ws: torch.Tensor, stream=None) -> None:
    """Softmax attention of one decode query per (layer, sequence, query head) over the cache rows."""
    _check(_L.tri_decode_attention(ctypes.byref(m), ctypes.byref(kv), _p(K), _p(V), _p(q), float(softmax_scale),
                                   _p(out), _p(lse), _p(ws), ws.numel() * ws.element_size(), _s(stream)),
           "tri_decode_attention")


def tri_decode_attention_tc(m: TriModel, kv: TriKvDesc, K: torch.Tensor, V: torch.Tensor, q: torch.Tensor,
                            softmax_scale: float, out: torch.Tensor, lse, ws: torch.Tensor, stream=None) -> None:
    """tri_decode_attention on the tensor-memory (tcgen05) kernel: bf16 contiguous caches, head dim 128, G <= 16."""
    _check(_L.tri_decode_attention_tc(ctypes.byref(m), ctypes.byref(kv), _p(K), _p(V), _p(q), float(softmax_scale),
                                      _p(out), _p(lse), _p(ws), ws.numel() * ws.element_size(), _s(stream)),
           "tri_decode_attention_tc")


def tri_score_compact(m: TriModel, kv: TriKvDesc, K: torch.Tensor, V: torch.Tensor, pos, centres: torch.Tensor,
                      mean_norm: torch.Tensor, p_now: torch.Tensor, offsets, key_mode: int, B: int, W: int,
                      max_row_len: int, out: TriOutDesc, K_out: torch.Tensor, V_out: torch.Tensor, pos_out,
                      kept_idx, kept_count, scores, ws: torch.Tensor, stream=None) -> None:
    """tri_score + tri_compact in one call, fused on chip when max_row_len <= TRI_FUSED_MAX_ROW."""
    offs = (ctypes.c_int32 * max(len(offsets), 1))(*[int(o) for o in offsets])
    _check(_L.tri_score_compact(ctypes.byref(m), ctypes.byref(kv), _p(K), _pd(V), _p(pos), _p(centres),
                                _p(mean_norm), _p(p_now), offs, len(offsets), int(key_mode), int(B), int(W),
                                int(max_row_len), ctypes.byref(out), _pd(K_out), _pd(V_out), _pd(pos_out),
                                _p(kept_idx), _p(kept_count), _p(scores), _p(ws), ws.numel() * ws.element_size(),
                                _s(stream)), "tri_score_compact")


def tri_status_check(ws: torch.Tensor, stream=None):
    """Synchronise, read and clear the device flag word.  Returns (status, flags)."""
    flags = ctypes.c_uint32(0)
    st = _L.tri_status_check(_p(ws), ctypes.byref(flags), _s(stream))
    return st, int(flags.value)


def tri_calib_save(path: str, m: TriModel, nq: int, centres: torch.Tensor, mean_norm: torch.Tensor) -> None:
    """Write a calibration file (model shape, nq and the centres bit for bit).  The
    centres may be on any device; they are copied to contiguous host float32
    tensors for the call (the library reads host memory here)."""
    c = centres.detach().to("cpu", torch.float32).contiguous()
    n = mean_norm.detach().to("cpu", torch.float32).contiguous()
    F = m.head_dim // 2
    if c.numel() != m.n_layers * m.n_q_heads * F * 2 or n.numel() != m.n_layers * m.n_q_heads * F:
        raise ValueError("centres / mean_norm do not match the model shape")
    _check(_L.tri_calib_save(str(path).encode(), ctypes.byref(m), int(nq), ctypes.c_void_p(c.data_ptr()),
                             ctypes.c_void_p(n.data_ptr())), "tri_calib_save")


def tri_calib_load(path: str, device=None):
    """Read a calibration file -> (model, nq, centres [L][Hq][d/2][2], mean_norm
    [L][Hq][d/2]) as float32 tensors on `device` (host when None)."""
    m = TriModel()
    nq = ctypes.c_int64(0)
    _check(_L.tri_calib_load(str(path).encode(), ctypes.byref(m), ctypes.byref(nq), None, None, 0),
           "tri_calib_load (header)")
    F = m.head_dim // 2
    c = torch.empty(m.n_layers, m.n_q_heads, F, 2, dtype=torch.float32)
    n = torch.empty(m.n_layers, m.n_q_heads, F, dtype=torch.float32)
    m2 = TriModel()
    _check(_L.tri_calib_load(str(path).encode(), ctypes.byref(m2), ctypes.byref(nq), ctypes.c_void_p(c.data_ptr()),
                             ctypes.c_void_p(n.data_ptr()), n.numel()), "tri_calib_load")
    if device is not None:
        c, n = c.to(device), n.to(device)
    return m2, int(nq.value), c, n


def tri_selftest_wait_timeout(ws: torch.Tensor, limit_ns: int, stream=None) -> None:
    """Enqueue the self-test of the staged kernels' bounded wait: one warp waits
    `limit_ns` on a barrier nothing completes and sets TRI_FLAG_STAGE_TIMEOUT
    (read it with ``tri_status_check``)."""
    _check(_L.tri_selftest_wait_timeout(_p(ws), ws.numel() * ws.element_size(), int(limit_ns), _s(stream)),
           "tri_selftest_wait_timeout")


def tri_score_noalloc(m: TriModel, kv: TriKvDesc, K: torch.Tensor, pos, centres: torch.Tensor,
                      mean_norm: torch.Tensor, p_now: torch.Tensor, offsets, key_mode: int,
                      scores: torch.Tensor, stream=None) -> None:
    """``tri_score`` for callers that cannot allocate device memory: the scratch is a
    fixed array inside the library (at most TRI_NOALLOC_MAX_ROWS rows; calls on a
    device share it, so calls that overlap on the GPU race)."""
    offs = (ctypes.c_int32 * max(len(offsets), 1))(*[int(o) for o in offsets])
    _check(_L.tri_score_noalloc(ctypes.byref(m), ctypes.byref(kv), _p(K), _p(pos), _p(centres),
                                _p(mean_norm), _p(p_now), offs, len(offsets), int(key_mode),
                                _p(scores), _s(stream)), "tri_score_noalloc")
