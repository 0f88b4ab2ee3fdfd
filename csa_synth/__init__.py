"""Seeded synthetic inputs for the CSA2 sparse-attention step.

This module is shared by the CPU oracle (``oracle/``), the tests and the
benchmark.  It draws random numbers and arranges them into the shapes of the
workloads; it contains none of the method's arithmetic (no FP4/FP8 encoding,
no scoring, no selection, no attention).  Both sides receive the same fp32 /
bf16 values from here and each side quantises them with its own code.

Every tensor is addressed by ``(seed, tensor_id)`` and split into chunks of
``CHUNK_ROWS`` rows; chunk ``c`` is drawn from
``numpy.random.default_rng(SeedSequence([seed, tensor_id, c]))``.  Any row
range can therefore be regenerated on its own, which lets the oracle rebuild
only the rows it samples from a cache that does not fit in host memory.
"""
from .gen import (
    CHUNK_ROWS,
    normal_rows,
    uniform_rows,
    gather_normal_rows,
    tid,
    outlier_channels,
    planted_positions,
    planted_key_row,
    TensorId,
)
from .configs import CONFIGS, Config, LayerSpec, get_config

__all__ = [
    "CHUNK_ROWS",
    "normal_rows",
    "uniform_rows",
    "outlier_channels",
    "planted_positions",
    "planted_key_row",
    "TensorId",
    "CONFIGS",
    "Config",
    "LayerSpec",
    "get_config",
]
