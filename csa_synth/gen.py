"""Chunked, seeded random tensors (no method arithmetic here).

A tensor is an endless sequence of rows of a fixed width.  Rows are grouped
into chunks of ``CHUNK_ROWS``; chunk ``c`` of tensor ``tid`` under ``seed`` is
drawn from ``default_rng(SeedSequence([seed, tid, c]))``.  The draws are
deterministic across machines (NumPy's PCG64 + ziggurat), so the oracle can
regenerate any row range on its own.
"""
from __future__ import annotations

import enum
from concurrent.futures import ThreadPoolExecutor

import numpy as np

CHUNK_ROWS = 4096


class TensorId(enum.IntEnum):
    """Base ids; a per-layer tensor uses ``(base << 8) | layer``."""

    MAIN_LATENT = 1     # main-KV latent rows, [B * T, 512] (owner layers)
    WINDOW_LATENT = 2   # sliding-window latent rows, [B * n_win_rows, 512]
    INDEX_KEY = 3       # indexer key rows, [B * T, 64] (owner layers)
    INDEX_QUERY = 4     # indexer query rows, [B * n_q * H_I, 64]
    INDEX_WEIGHT = 5    # indexer head weights, [B * n_q, H_I]
    ATTN_QUERY = 6      # attention query rows, [B * n_q * H, 512]
    OUTLIER = 7         # outlier channel choice
    PLANT = 8           # planted-position offsets
    SINK = 9            # optional per-head sink logits
    SCORES = 10         # synthetic score rows for selection tests
    MAIN_GATE = 11      # compressor gate logits of main-KV token rows, [B * T, 512] (m > 1 owners)
    INDEX_GATE = 12     # compressor gate logits of indexer-key token rows, [B * T, 64]


def tid(base: TensorId, layer: int = 0) -> int:
    return (int(base) << 8) | int(layer)


def _chunk(seed: int, t: int, c: int, width: int, kind: str) -> np.ndarray:
    rng = np.random.default_rng(np.random.SeedSequence([int(seed), int(t), int(c)]))
    if kind == "normal":
        return rng.standard_normal((CHUNK_ROWS, width), dtype=np.float32)
    if kind == "uniform":
        return rng.random((CHUNK_ROWS, width), dtype=np.float32)
    raise ValueError(kind)


def _rows(seed, t, row0, nrows, width, kind, threads):
    out = np.empty((nrows, width), dtype=np.float32)
    if nrows == 0:
        return out
    c0 = row0 // CHUNK_ROWS
    c1 = (row0 + nrows - 1) // CHUNK_ROWS

    def fill(c):
        blk = _chunk(seed, t, c, width, kind)
        lo = max(row0, c * CHUNK_ROWS)
        hi = min(row0 + nrows, (c + 1) * CHUNK_ROWS)
        out[lo - row0:hi - row0] = blk[lo - c * CHUNK_ROWS:hi - c * CHUNK_ROWS]

    chunks = range(c0, c1 + 1)
    if threads > 1 and c1 > c0:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, chunks))
    else:
        for c in chunks:
            fill(c)
    return out


def normal_rows(seed: int, t: int, row0: int, nrows: int, width: int,
                threads: int = 1) -> np.ndarray:
    """Rows ``[row0, row0 + nrows)`` of an N(0,1) fp32 tensor of ``width`` columns."""
    return _rows(seed, t, row0, nrows, width, "normal", threads)


def uniform_rows(seed: int, t: int, row0: int, nrows: int, width: int,
                 threads: int = 1) -> np.ndarray:
    """Rows of a U[0,1) fp32 tensor."""
    return _rows(seed, t, row0, nrows, width, "uniform", threads)


def gather_normal_rows(seed: int, t: int, rows: np.ndarray, width: int) -> np.ndarray:
    """Arbitrary (possibly repeated) rows of an N(0,1) tensor, by chunk."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.size, width), dtype=np.float32)
    if rows.size == 0:
        return out
    chunk_of = rows // CHUNK_ROWS
    for c in np.unique(chunk_of):
        sel = np.nonzero(chunk_of == c)[0]
        blk = _chunk(seed, t, int(c), width, "normal")
        out[sel] = blk[rows[sel] - c * CHUNK_ROWS]
    return out


def outlier_channels(seed: int, dim: int = 512, fraction: float = 0.01) -> np.ndarray:
    """Channel indices (sorted) that a config scales up; count = round(fraction*dim)."""
    n = int(round(fraction * dim))
    rng = np.random.default_rng(np.random.SeedSequence([int(seed), int(TensorId.OUTLIER)]))
    return np.sort(rng.choice(dim, size=n, replace=False)).astype(np.int64)


def planted_positions(seed: int, b: int, T: int, stride: int = 4096) -> np.ndarray:
    """One planted position per ``stride`` positions: stride*i + U{0..stride-1}."""
    n = T // stride
    rng = np.random.default_rng(np.random.SeedSequence([int(seed), int(TensorId.PLANT), int(b)]))
    off = rng.integers(0, stride, size=n)
    return (np.arange(n, dtype=np.int64) * stride + off).astype(np.int64)


def planted_key_row(q_rows: np.ndarray, w: np.ndarray, gain: float = 4.0) -> np.ndarray:
    """An fp32 key row aligned with the head-weighted query direction.

    ``q_rows``: fp32 [H_I, d] pre-quantisation indexer queries of the layer that
    builds the pool, ``w``: fp32 [H_I] head weights.  Returns
    ``gain * v / rms(v)`` with ``v = sum_j w_j q_j``.  This only shapes the
    synthetic key distribution (positions that the indexer should rank high);
    each side still encodes the row itself.
    """
    v = (w.astype(np.float64)[:, None] * q_rows.astype(np.float64)).sum(axis=0)
    rms = np.sqrt(np.mean(v * v))
    return (gain * v / rms).astype(np.float32)
