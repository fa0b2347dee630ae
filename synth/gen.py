"""Seeded synthetic KV caches with concentrated pre-RoPE centres.

This module plays the model that wrote the cache.  It holds none of the
scoring, selection or compaction arithmetic; both the CUDA path and the CPU
oracle consume what it produces (the oracle through the exact bf16 bits).

Generator (the concentrated-centre premise of "TriAttention：基于三角函数 KV
压缩的高效长推理", section 核心洞见: pre-RoPE Q and K cluster around fixed,
position-stable centres):
  * per (layer, KV head) and pair f, a centre mu_f with magnitude
    exp(N(0,1)) and phase U[0, 2pi);
  * pre-RoPE key pairs k_f = mu_f + eps, eps real and imaginary parts i.i.d.
    N(0, (r |mu_f|)^2), r the head's noise ratio;
  * keys are RoPE-rotated at their position (pairs (f, f+d/2) for
    rotate-half RoPE, (2f, 2f+1) for interleaved RoPE; w_f = theta^(-2f/d),
    angles reduced in fp64) and rounded to bf16;
  * calibration queries: every query head draws its own centres and ratio and
    its pre-RoPE queries the same way (not rotated);
  * values are i.i.d. N(0, 1) in bf16;
  * zero-centre heads keep their drawn |mu| for the noise scale but set the
    centre itself to 0, so their keys are pure noise (their query heads too).
Randomness comes from torch generators seeded by a hash of (seed, workload,
layer, component), so any layer can be regenerated alone.
"""
from __future__ import annotations

import hashlib
import math
from dataclasses import dataclass

import numpy as np
import torch

from .workloads import Workload


def _seed(*parts) -> int:
    h = hashlib.sha256(repr(parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*parts))
    return g


_ROT_CACHE: dict = {}


def rotation(positions: torch.Tensor, theta: float, d: int):
    """(cos, sin) fp32 [n][d/2] of the RoPE angles w_f * p, reduced in fp64."""
    dev = positions.device
    F = d // 2
    w = torch.pow(torch.tensor(float(theta), dtype=torch.float64, device=dev),
                  -2.0 * torch.arange(F, dtype=torch.float64, device=dev) / d)
    a = torch.remainder(positions.to(torch.float64)[:, None] * w[None, :], 2.0 * math.pi)
    return torch.cos(a).to(torch.float32), torch.sin(a).to(torch.float32)


def _rotation_arange(n: int, theta: float, d: int, device):
    key = (n, theta, d, str(device))
    if key not in _ROT_CACHE:
        if len(_ROT_CACHE) > 4:
            _ROT_CACHE.clear()
        _ROT_CACHE[key] = rotation(torch.arange(n, device=device), theta, d)
    return _ROT_CACHE[key]


@dataclass
class LayerHeads:
    """Centres and noise scales of one layer (complex values as re/im fp32 pairs)."""
    key_re: torch.Tensor  # [H][F]
    key_im: torch.Tensor
    key_scale: torch.Tensor  # [H][F]  r_h * |mu_{h,f}|
    q_re: torch.Tensor  # [Hq][F]
    q_im: torch.Tensor
    q_scale: torch.Tensor  # [Hq][F]
    zero: np.ndarray  # [H] bool


def layer_heads(wl: Workload, layer: int, device) -> LayerHeads:
    g = _gen(device, wl.seed, wl.name, "heads", layer)
    H, Hq, F = wl.n_kv_heads, wl.n_q_heads, wl.head_dim // 2
    lo, hi = wl.noise

    def centres(n):
        mag = torch.exp(torch.randn(n, F, generator=g, device=device))
        ph = torch.rand(n, F, generator=g, device=device) * (2.0 * math.pi)
        r = lo + (hi - lo) * torch.rand(n, 1, generator=g, device=device)
        return mag * torch.cos(ph), mag * torch.sin(ph), r * mag

    kre, kim, ksc = centres(H)
    qre, qim, qsc = centres(Hq)
    zero = wl.zero_centre_pairs()[layer]
    if zero.any():
        zk = torch.as_tensor(zero, device=device)
        zq = zk.repeat_interleave(wl.group)
        kre[zk] = 0.0
        kim[zk] = 0.0
        qre[zq] = 0.0
        qim[zq] = 0.0
    return LayerHeads(kre, kim, ksc, qre, qim, qsc, zero)


def place_pairs(out: torch.Tensor, re: torch.Tensor, im: torch.Tensor, interleaved: bool) -> torch.Tensor:
    """Write pair values into the last dim of ``out``: (f, f+d/2) or (2f, 2f+1)."""
    F = out.shape[-1] // 2
    if interleaved:
        out[..., 0::2] = re
        out[..., 1::2] = im
    else:
        out[..., :F] = re
        out[..., F:] = im
    return out


def head_keys(heads: LayerHeads, h: int, positions: torch.Tensor, g: torch.Generator,
              theta: float, d: int, rotate: bool = True, arange_n: int = 0,
              interleaved: bool = False) -> torch.Tensor:
    """Keys of KV head h at ``positions``: bf16 [n][d] (RoPE'd unless rotate=False)."""
    n = positions.shape[0]
    F = d // 2
    dev = positions.device
    er = torch.randn(n, F, generator=g, device=dev)
    ei = torch.randn(n, F, generator=g, device=dev)
    kr = heads.key_re[h][None, :] + heads.key_scale[h][None, :] * er
    ki = heads.key_im[h][None, :] + heads.key_scale[h][None, :] * ei
    if rotate:
        c, s = _rotation_arange(arange_n, theta, d, dev) if arange_n else rotation(positions, theta, d)
        c, s = c[:n], s[:n]
        kr, ki = kr * c - ki * s, kr * s + ki * c
    return place_pairs(torch.empty(n, d, dtype=torch.bfloat16, device=dev), kr, ki, interleaved)


def calib_queries(wl: Workload, layer: int, device, heads: LayerHeads = None) -> torch.Tensor:
    """Pre-RoPE calibration queries of one layer: bf16 [Hq][n_calib][d]."""
    heads = heads if heads is not None else layer_heads(wl, layer, device)
    g = _gen(device, wl.seed, wl.name, "queries", layer)
    Hq, F, n = wl.n_q_heads, wl.head_dim // 2, wl.n_calib
    er = torch.randn(Hq, n, F, generator=g, device=device)
    ei = torch.randn(Hq, n, F, generator=g, device=device)
    out = torch.empty(Hq, n, wl.head_dim, dtype=torch.bfloat16, device=device)
    return place_pairs(out, heads.q_re[:, None, :] + heads.q_scale[:, None, :] * er,
                       heads.q_im[:, None, :] + heads.q_scale[:, None, :] * ei, wl.interleaved)


@dataclass
class ContigCache:
    """Rows (layer, sequence, KV head) laid end to end: row r holds keys
    row_off[r] .. row_off[r+1]-1 of K/V/pos."""
    wl: Workload
    layers: list
    lens: np.ndarray  # [S] int64
    K: torch.Tensor  # bf16 [total][d]
    V: torch.Tensor  # bf16 [total][d] (or None)
    pos: torch.Tensor  # int32 [total]
    row_off: torch.Tensor  # int64 [R+1] on the cache's device
    row_off_np: np.ndarray
    p_now: torch.Tensor  # int64 [S]
    qcal: torch.Tensor  # bf16 [L][Hq][n_calib][d]

    @property
    def n_rows(self) -> int:
        return len(self.row_off_np) - 1

    @property
    def total(self) -> int:
        return int(self.row_off_np[-1])

    def row_lhs(self, r: int):
        """(layer index into ``layers``, sequence, KV head) of row r."""
        H, S = self.wl.n_kv_heads, len(self.lens)
        return r // (S * H), (r // H) % S, r % H


def contig_row_offsets(n_layers: int, lens: np.ndarray, H: int) -> np.ndarray:
    per_row = np.tile(np.repeat(np.asarray(lens, dtype=np.int64), H), n_layers)
    return np.concatenate([[0], np.cumsum(per_row)]).astype(np.int64)


def make_contig(wl: Workload, device, layers=None, lens=None, with_values: bool = True,
                rotate: bool = True) -> ContigCache:
    layers = list(range(wl.n_layers)) if layers is None else list(layers)
    lens = wl.seq_lengths() if lens is None else np.asarray(lens, dtype=np.int64)
    H, d = wl.n_kv_heads, wl.head_dim
    row_off = contig_row_offsets(len(layers), lens, H)
    total = int(row_off[-1])
    K = torch.empty(total, d, dtype=torch.bfloat16, device=device)
    V = torch.empty(total, d, dtype=torch.bfloat16, device=device) if with_values else None
    pos = torch.empty(total, dtype=torch.int32, device=device)
    qcal = torch.empty(len(layers), wl.n_q_heads, wl.n_calib, d, dtype=torch.bfloat16,
                       device=device)
    nmax = int(lens.max()) if len(lens) else 0
    r = 0
    for li, layer in enumerate(layers):
        heads = layer_heads(wl, layer, device)
        qcal[li] = calib_queries(wl, layer, device, heads)
        gk = _gen(device, wl.seed, wl.name, "keys", layer)
        gv = _gen(device, wl.seed, wl.name, "values", layer)
        for s, n in enumerate(lens):
            n = int(n)
            p = torch.arange(n, device=device)
            for h in range(H):
                a, b = int(row_off[r]), int(row_off[r + 1])
                if n:
                    K[a:b] = head_keys(heads, h, p, gk, wl.theta, d, rotate, arange_n=nmax,
                                       interleaved=wl.interleaved)
                    if V is not None:
                        V[a:b] = torch.randn(n, d, generator=gv, device=device).to(torch.bfloat16)
                    pos[a:b] = p.to(torch.int32)
                r += 1
    return ContigCache(wl, layers, lens, K, V, pos, torch.as_tensor(row_off, device=device),
                       row_off, torch.as_tensor(lens, device=device), qcal)


@dataclass
class PagedCache:
    """vLLM-style paged cache of one layer: K/V [n_blocks][block][H][d], pos
    [n_blocks][block][H]; sequence s owns blocks block_table[s][0 .. ceil(len/block)-1]."""
    wl: Workload
    lens: np.ndarray
    K: torch.Tensor
    V: torch.Tensor
    pos: torch.Tensor
    block_table: torch.Tensor  # int32 [S][max_blocks]
    block_table_np: np.ndarray
    p_now: torch.Tensor


def paged_row_offsets(lens: np.ndarray, H: int) -> np.ndarray:
    """Score-buffer offsets of rows (sequence, KV head) of one paged layer."""
    return contig_row_offsets(1, lens, H)


def make_paged(wl: Workload, device, layer: int = 0, lens=None, max_blocks: int = None,
               n_blocks: int = None) -> PagedCache:
    lens = wl.seq_lengths() if lens is None else np.asarray(lens, dtype=np.int64)
    H, d, bs = wl.n_kv_heads, wl.head_dim, wl.block_size
    need = [(int(n) + bs - 1) // bs for n in lens]
    max_blocks = max_blocks or max(need)
    n_blocks = n_blocks or sum(need)
    rng = np.random.default_rng([wl.seed, 3, layer, len(lens)])
    perm = rng.permutation(n_blocks)
    table = np.full((len(lens), max_blocks), -1, dtype=np.int32)
    c = 0
    for s, nb in enumerate(need):
        table[s, :nb] = perm[c:c + nb]
        c += nb
    K = torch.zeros(n_blocks, bs, H, d, dtype=torch.bfloat16, device=device)
    V = torch.zeros(n_blocks, bs, H, d, dtype=torch.bfloat16, device=device)
    pos = torch.full((n_blocks, bs, H), -1, dtype=torch.int32, device=device)
    heads = layer_heads(wl, layer, device)
    gk = _gen(device, wl.seed, wl.name, "keys", layer)
    gv = _gen(device, wl.seed, wl.name, "values", layer)
    nmax = int(lens.max())
    tt = torch.as_tensor(table, device=device, dtype=torch.int64)
    for s, n in enumerate(lens):
        n = int(n)
        p = torch.arange(n, device=device)
        blk = tt[s, p // bs]
        slot = p % bs
        for h in range(H):
            K[blk, slot, h] = head_keys(heads, h, p, gk, wl.theta, d, True, arange_n=nmax,
                                        interleaved=wl.interleaved)
            V[blk, slot, h] = torch.randn(n, d, generator=gv, device=device).to(torch.bfloat16)
            pos[blk, slot, h] = p.to(torch.int32)
    return PagedCache(wl, lens, K, V, pos, torch.as_tensor(table, device=device), table,
                      torch.as_tensor(lens, device=device))


def decode_keys(wl: Workload, layer: int, round_idx: int, start: np.ndarray, count: int,
                device):
    """New decode tokens of every sequence: keys and values bf16 [S][count][H][d] at
    positions start[s] .. start[s]+count-1 (RoPE'd), from the layer's centres."""
    heads = layer_heads(wl, layer, device)
    g = _gen(device, wl.seed, wl.name, "decode", layer, round_idx)
    S, H, d = len(start), wl.n_kv_heads, wl.head_dim
    Kn = torch.empty(S, count, H, d, dtype=torch.bfloat16, device=device)
    Vn = torch.empty(S, count, H, d, dtype=torch.bfloat16, device=device)
    for s in range(S):
        p = torch.arange(int(start[s]), int(start[s]) + count, device=device)
        for h in range(H):
            Kn[s, :, h] = head_keys(heads, h, p, g, wl.theta, d, True, interleaved=wl.interleaved)
            Vn[s, :, h] = torch.randn(count, d, generator=g, device=device).to(torch.bfloat16)
    return Kn, Vn


FP8_MAX = 448.0  # largest finite OCP e4m3 value


def to_fp8(t: torch.Tensor, chunk: int = 1 << 28) -> torch.Tensor:
    """The cache as an fp8 e4m3 cache would store it: clamp to +-448, round to nearest.
    Converted `chunk` elements at a time, so a cache near the device's size needs no
    full-size fp32 copy."""
    out = torch.empty(t.shape, dtype=torch.float8_e4m3fn, device=t.device)
    src, dst = t.reshape(-1), out.view(-1)
    for i in range(0, src.numel(), chunk):
        dst[i:i + chunk] = src[i:i + chunk].float().clamp_(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn)
    return out


def decode_queries(wl: Workload, layer: int, p_now: np.ndarray, device, heads: LayerHeads = None) -> torch.Tensor:
    """The next token's queries of every sequence: bf16 [S][Hq][d], drawn from the
    layer's query centres like the calibration queries and RoPE-rotated at the
    sequence's position p_now[s] (the position being decoded)."""
    heads = heads if heads is not None else layer_heads(wl, layer, device)
    g = _gen(device, wl.seed, wl.name, "decode_queries", layer)
    S, Hq, F, d = len(p_now), wl.n_q_heads, wl.head_dim // 2, wl.head_dim
    er = torch.randn(S, Hq, F, generator=g, device=device)
    ei = torch.randn(S, Hq, F, generator=g, device=device)
    qr = heads.q_re[None] + heads.q_scale[None] * er
    qi = heads.q_im[None] + heads.q_scale[None] * ei
    c, s = rotation(torch.as_tensor(np.asarray(p_now), device=device), wl.theta, d)  # [S][F]
    c, s = c[:, None, :], s[:, None, :]
    out = torch.empty(S, Hq, d, dtype=torch.bfloat16, device=device)
    return place_pairs(out, qr * c - qi * s, qr * s + qi * c, wl.interleaved)
