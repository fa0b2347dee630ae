"""The five synthetic KV-cache workloads, by shape.

Each stands in for a real model's cache: Qwen3-8B has 36 layers, 32 query
heads and 8 KV heads of dim 128 with RoPE theta 1e6; Qwen3-32B has 64 layers,
64 query heads and 8 KV heads.  No dataset or weights are used: keys and
queries come from the concentrated-centre generator in ``synth.gen``.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    batch: int
    seq_len: tuple  # (lo, hi) inclusive; lo == hi for a fixed length
    budget: int  # B: keys kept per (layer, sequence, KV head), window included
    window: int  # W: most recent slots always kept
    n_offsets: int  # future offsets 1, 2, 4, ..., 2^(n_offsets-1)
    noise: tuple = (0.3, 0.3)  # per-head noise ratio r, uniform in [lo, hi]
    zero_centre_frac: float = 0.0  # share of (layer, KV head) pairs with zero centres
    layout: str = "contig"  # "contig" | "paged"
    block_size: int = 16
    rescore_every: int = 0  # paged decode rounds: new tokens per round
    rounds: int = 0
    head_dim: int = 128
    rope_style: str = "half"  # "half": pair f = dims (f, f+d/2); "interleaved": (2f, 2f+1)
    theta: float = 1e6
    n_calib: int = 1024  # calibration queries per query head
    seed: int = 20261202

    @property
    def offsets(self) -> list:
        return [2 ** e for e in range(self.n_offsets)]

    @property
    def interleaved(self) -> bool:
        return self.rope_style == "interleaved"

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def seq_lengths(self) -> np.ndarray:
        lo, hi = self.seq_len
        if lo == hi:
            return np.full(self.batch, lo, dtype=np.int64)
        rng = np.random.default_rng([self.seed, 1, self.batch, lo, hi])
        return rng.integers(lo, hi + 1, size=self.batch).astype(np.int64)

    def zero_centre_pairs(self) -> np.ndarray:
        """Boolean [n_layers][n_kv_heads]: heads whose centres are zero (pure noise)."""
        m = np.zeros((self.n_layers, self.n_kv_heads), dtype=bool)
        k = int(round(self.zero_centre_frac * m.size))
        if k:
            rng = np.random.default_rng([self.seed, 2, m.size])
            m.reshape(-1)[rng.permutation(m.size)[:k]] = True
        return m

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # one layer, 8 KV heads x 4 query heads, 4096 keys, B=512, W=64, 13 offsets
    "single_layer_4k": Workload("single_layer_4k", 1, 32, 8, 1, (4096, 4096), 512, 64, 13),
    # Qwen3-8B-shaped cache, 32K keys per head, B=2048, W=128, 13 offsets
    "qwen3_8b_32k": Workload("qwen3_8b_32k", 36, 32, 8, 1, (32768, 32768), 2048, 128, 13),
    # paged batch: 16 sequences of 8K..32K keys in 16-token blocks, one layer of the
    # single-layer shape; re-scored after every 128 decode tokens against the
    # retained 2048
    "paged_16seq": Workload("paged_16seq", 1, 32, 8, 16, (8192, 32768), 2048, 128, 13,
                            layout="paged", rescore_every=128, rounds=8),
    # Qwen3-32B-shaped cache, 128K keys, batch 4, B=4096, W=256, 17 offsets,
    # noise ratio uniform in [0.1, 0.8] per head
    "qwen3_32b_128k": Workload("qwen3_32b_128k", 64, 64, 8, 4, (131072, 131072), 4096, 256, 17,
                               noise=(0.1, 0.8)),
    # steady-state sweep: batch 64, lengths 4K..64K, Qwen3-8B shape, B in {1024, 2048, 4096}
    "sweep_b64": Workload("sweep_b64", 36, 32, 8, 64, (4096, 65536), 2048, 128, 13),
    # the same with 5% of (layer, KV head) pairs given zero-magnitude centres
    "sweep_b64_adversarial": Workload("sweep_b64_adversarial", 36, 32, 8, 64, (4096, 65536), 2048,
                                      128, 13, zero_centre_frac=0.05),
}
SWEEP_BUDGETS = (1024, 2048, 4096)
