"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This package holds no arithmetic of the attention method itself: it only
draws the FP16 keys, values and queries of the synthetic workloads
(LLaMA-3.1-8B-shaped decode attention, 8K-128K context) from a
counter-based generator, so that any (layer, batch, kv-head, token range)
slice can be regenerated on its own, bit-identically on the CPU and on a
CUDA device.
"""

from .gen import (  # noqa: F401
    WORKLOADS,
    Workload,
    default_thresholds,
    kv_unit,
    kv_row,
    kv_layer,
    row_lengths,
    queries,
    outlier_channels,
    plant_positions,
    hash32,
)
