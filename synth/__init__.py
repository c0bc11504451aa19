"""Seeded synthetic inputs for the SAGA + Atop-N decode attention step.

Shared by the tests, the benchmark and the oracle's checks. It draws random
inputs and nothing else: no attention arithmetic lives here.
"""
from .philox import philox4x32_10
from .normal import box_muller
from .workload import (WORKLOADS, Workload, F32, BF16, cache, cache_rows, cache_rows_at,
                       normals, planted, queries, seq_lens, to_storage,
                       unit_direction, widen)

__all__ = ["philox4x32_10", "box_muller", "WORKLOADS", "Workload", "F32", "cache_rows_at",
           "BF16", "cache", "cache_rows", "normals", "planted", "queries",
           "seq_lens", "to_storage", "unit_direction", "widen"]
