"""Shared helpers of the GPU parity tests and the benchmark's CPU leg.

Oracle inputs are always the generator's bits (read back from wherever the
generator put them) or oracle outputs; nothing computed by the CUDA path is
ever fed to the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy()


def raw_bits(t: torch.Tensor) -> np.ndarray:
    """Stored bits of a K/V tensor: int16 per bf16 element, uint8 per fp8 element."""
    if t.dtype == torch.float8_e4m3fn:
        return t.detach().contiguous().view(torch.uint8).cpu().numpy()
    return bits16(t)


def torch_bits(t: torch.Tensor) -> torch.Tensor:
    """The stored bits of a bf16/fp8 tensor as an integer tensor (for exact comparison)."""
    return t.view(torch.uint8) if t.dtype == torch.float8_e4m3fn else t.view(torch.int16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16 or fp8 e4m3 tensor's bits to float64 (host)."""
    if t.dtype == torch.float8_e4m3fn:
        return oracle.e4m3_bits_to_f64(raw_bits(t))
    return oracle.bf16_bits_to_f64(bits16(t))


def oracle_calibration(qcal: torch.Tensor, interleaved: bool = False):
    """Oracle calibration of queries bf16 [L][Hq][nq][d] -> (centres fp64 [L][Hq][F][2],
    mnorm fp64 [L][Hq][F])."""
    L, Hq, nq, d = qcal.shape
    q = to_f64(qcal).reshape(L, Hq, nq, d)
    cs = np.empty((L, Hq, d // 2, 2))
    ms = np.empty((L, Hq, d // 2))
    for l in range(L):
        for g in range(Hq):
            cs[l, g], ms[l, g] = oracle.calib(q[l, g], interleaved=interleaved)
    return cs, ms


def as_f32_exact(a: np.ndarray) -> np.ndarray:
    """Round to fp32 and widen back: the values both sides then see."""
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def pair_norms(keys: np.ndarray, interleaved: bool = False) -> np.ndarray:
    """|k_f| per key and pair: dims (f, f+d/2), or (2f, 2f+1) when interleaved."""
    F = keys.shape[1] // 2
    if interleaved:
        return np.hypot(keys[:, 0::2], keys[:, 1::2])
    return np.hypot(keys[:, :F], keys[:, F:])


def series_bound(theta, centres_l, mnorms_l, h, G, keys, offsets, interleaved=False) -> np.ndarray:
    """Absolute-value bound M_j = sum_f (|A_f| + |c_f|) |k_f| of a row's score series
    (the scale the score tolerance is relative to; scores can cancel near 0)."""
    d = keys.shape[1]
    F = d // 2
    w = np.power(float(theta), -2.0 * np.arange(F) / d)
    S = np.exp(1j * np.outer(np.asarray(offsets, dtype=np.float64), w)).sum(axis=0)
    qb = centres_l[h * G:(h + 1) * G]
    qc = qb[..., 0] + 1j * qb[..., 1]
    Q = qc.mean(axis=0)
    c = (mnorms_l[h * G:(h + 1) * G] - np.abs(qc)).mean(axis=0)
    kn = pair_norms(keys, interleaved)
    return kn @ (np.abs(Q) * np.abs(S) + np.abs(c))


def score_error(gpu: np.ndarray, ref: np.ndarray, bound: np.ndarray) -> float:
    """max_j |gpu_j - ref_j| / M_j (bound floored to avoid 0/0 on all-zero keys)."""
    return float(np.max(np.abs(gpu - ref) / np.maximum(bound, 1e-30))) if len(ref) else 0.0


def check_kept_within_ties(kept_gpu, ref_scores, B, W, bound, rtol=1e-5):
    """Selection parity with the boundary-tie allowance: the GPU's kept set may differ
    from the oracle's only at slots whose oracle score is within rtol of the oracle's
    threshold t (the (B-W)-th best non-window score), relative to max(|t|, M_j)."""
    n = len(ref_scores)
    kept_gpu = np.asarray(kept_gpu, dtype=np.int64)
    ref = oracle.select(ref_scores, B, W)
    assert len(kept_gpu) == len(ref) == min(n, B)
    assert np.all(np.diff(kept_gpu) > 0)
    if n <= B:
        np.testing.assert_array_equal(kept_gpu, np.arange(n))
        return 0
    assert set(range(n - W, n)) <= set(kept_gpu.tolist())
    diff = np.setxor1d(kept_gpu, ref)
    if len(diff) == 0:
        return 0
    M = n - W
    cand = ref[ref < M]
    t = ref_scores[cand].min() if len(cand) else np.inf
    scale = np.maximum(abs(t), bound[diff])
    bad = diff[np.abs(ref_scores[diff] - t) > rtol * scale]
    assert len(bad) == 0, f"selection differs beyond ties at slots {bad[:10]}"
    return len(diff)
