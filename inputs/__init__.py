"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This package generates operator INPUTS only (geometry, edge features, node
features, weights, output cotangents). It holds none of the convolution's
arithmetic, imports neither the CUDA path nor the oracle, and is the one module
both sides see.
"""
from .workloads import (CONFIGS, LUNATP_CASES, SOBEK_COUNTS, SOBEK_DEGREES, Workload,  # noqa: F401
                        make_workload, sobek_count_graph, sobek_degree_graph, sobek_workload)
