"""Per-config input tensors as fp32 host arrays (values only; no encoding).

Row addressing: a per-sequence tensor with R rows per sequence keeps sequence
``b``'s row ``r`` at global row ``b * R + r`` of its chunked stream, so any
(b, row range) or scattered row set can be rebuilt independently.
"""
from __future__ import annotations

import numpy as np

from .configs import Config
from .gen import (TensorId, tid, normal_rows, uniform_rows, gather_normal_rows,
                  outlier_channels, planted_positions, planted_key_row)

try:  # bf16 rounding of the prefill latents (round to nearest even)
    import ml_dtypes as _mld
except ImportError:  # pragma: no cover
    _mld = None


def _to_bf16_values(x: np.ndarray) -> np.ndarray:
    if _mld is None:
        raise RuntimeError("ml_dtypes is required for bf16 latents")
    return x.astype(_mld.bfloat16).astype(np.float32)


def _shape_latents(cfg: Config, x: np.ndarray) -> np.ndarray:
    if cfg.outliers:
        ch = outlier_channels(cfg.seed, cfg.D)
        x[:, ch] *= np.float32(cfg.outlier_gain)
    if cfg.bf16_latents:
        x = _to_bf16_values(x)
    return x


def main_latent(cfg: Config, owner: int, b: int, t0: int, n: int, threads: int = 1) -> np.ndarray:
    """fp32 [n, D] main-KV latents of positions [t0, t0+n) of sequence b."""
    x = normal_rows(cfg.seed, tid(TensorId.MAIN_LATENT, owner), b * cfg.T + t0, n, cfg.D, threads)
    return _shape_latents(cfg, x)


def main_latent_at(cfg: Config, owner: int, b: int, positions: np.ndarray) -> np.ndarray:
    """fp32 [len(positions), D] main-KV latents at scattered positions."""
    rows = b * cfg.T + np.asarray(positions, dtype=np.int64)
    x = gather_normal_rows(cfg.seed, tid(TensorId.MAIN_LATENT, owner), rows, cfg.D)
    return _shape_latents(cfg, x)


def main_gate(cfg: Config, owner: int, b: int, t0: int, n: int, threads: int = 1) -> np.ndarray:
    """fp32 [n, D] compressor gate logits of token rows [t0, t0+n) (owners with m > 1), N(0, 2^2)."""
    return normal_rows(cfg.seed, tid(TensorId.MAIN_GATE, owner), b * cfg.T + t0, n, cfg.D, threads) * np.float32(2)


def main_gate_at(cfg: Config, owner: int, b: int, positions: np.ndarray) -> np.ndarray:
    """fp32 [len(positions), D] gate logits at scattered token rows."""
    rows = b * cfg.T + np.asarray(positions, dtype=np.int64)
    return gather_normal_rows(cfg.seed, tid(TensorId.MAIN_GATE, owner), rows, cfg.D) * np.float32(2)


def index_gate(cfg: Config, owner: int, b: int, t0: int, n: int, threads: int = 1) -> np.ndarray:
    """fp32 [n, d_I] compressor gate logits of indexer-key token rows, N(0, 2^2)."""
    return normal_rows(cfg.seed, tid(TensorId.INDEX_GATE, owner), b * cfg.T + t0, n, cfg.d_I, threads) * np.float32(2)


def window_latent(cfg: Config, layer: int, b: int) -> np.ndarray:
    """fp32 [win_rows, D] sliding-window latents of one layer and sequence."""
    R = cfg.win_rows
    x = normal_rows(cfg.seed, tid(TensorId.WINDOW_LATENT, layer), b * R, R, cfg.D)
    return _shape_latents(cfg, x)


def index_query(cfg: Config, layer: int, b: int) -> np.ndarray:
    """fp32 [n_q, H_I, d_I] indexer queries (before FP8 encoding)."""
    R = cfg.n_q * cfg.H_I
    x = normal_rows(cfg.seed, tid(TensorId.INDEX_QUERY, layer), b * R, R, cfg.d_I)
    return x.reshape(cfg.n_q, cfg.H_I, cfg.d_I)


def index_weight(cfg: Config, layer: int, b: int) -> np.ndarray:
    """fp32 [n_q, H_I] indexer head weights, U[0,1)."""
    return uniform_rows(cfg.seed, tid(TensorId.INDEX_WEIGHT, layer), b * cfg.n_q, cfg.n_q, cfg.H_I)


def attn_query(cfg: Config, layer: int, b: int) -> np.ndarray:
    """fp32 [n_q, H, D] attention queries."""
    R = cfg.n_q * cfg.H
    x = normal_rows(cfg.seed, tid(TensorId.ATTN_QUERY, layer), b * R, R, cfg.D)
    return x.reshape(cfg.n_q, cfg.H, cfg.D)


def plant_layer(cfg: Config) -> int:
    """The layer whose indexer queries define the planted key direction (the pool builder)."""
    for i, l in enumerate(cfg.layers):
        if l.build_pool:
            return i
    return 0


def planted(cfg: Config, b: int):
    """(positions, fp32 key row) planted into sequence b, or (empty, None)."""
    if not cfg.planted:
        return np.zeros(0, dtype=np.int64), None
    pos = planted_positions(cfg.seed, b, cfg.T, cfg.plant_stride)
    L = plant_layer(cfg)
    q = index_query(cfg, L, b)[-1]          # [H_I, d_I] of the last query token
    w = index_weight(cfg, L, b)[-1]         # [H_I]
    return pos, planted_key_row(q, w)


def index_key(cfg: Config, owner: int, b: int, t0: int, n: int, threads: int = 1) -> np.ndarray:
    """fp32 [n, d_I] indexer keys of positions [t0, t0+n), planted rows included."""
    x = normal_rows(cfg.seed, tid(TensorId.INDEX_KEY, owner), b * cfg.T + t0, n, cfg.d_I, threads)
    if cfg.planted:
        pos, row = planted(cfg, b)
        m = (pos >= t0) & (pos < t0 + n)
        x[pos[m] - t0] = row
    return x


def sink(cfg: Config, layer: int) -> np.ndarray:
    """fp32 [H] per-head sink logits (only used when a test enables sinks)."""
    return normal_rows(cfg.seed, tid(TensorId.SINK, layer), 0, 1, cfg.H)[0]
