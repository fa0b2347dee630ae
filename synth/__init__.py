"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

Holds the workload shapes and the concentrated-centre cache generator only;
no scoring, selection or compaction arithmetic lives here.
"""
from .workloads import SWEEP_BUDGETS, WORKLOADS, Workload  # noqa: F401
from .gen import (ContigCache, PagedCache, calib_queries, contig_row_offsets,  # noqa: F401
                  decode_keys, decode_queries, layer_heads, make_contig, make_paged, paged_row_offsets,
                  to_fp8)
