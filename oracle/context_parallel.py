"""Decode of one long sequence split across ranks by position (oracle; test
infrastructure only).

This is the exchange a context-parallel decode needs when one sequence's cache
is too long for one GPU.  The cache positions [0, T) are split into contiguous
shards, one per rank.  Each rank scores its own shard and keeps a local Top-K.
The global Top-K is the K best of the union of the local ones, ranked by score
descending, then position ascending.  This is exact: an element of the global
Top-K is among the best K of its own shard, since anything that beats it in
its shard beats it globally too.  Each rank then attends over the selected
entries that lie in its shard; the window entries belong to the rank that
holds the newest positions.  The partial results combine by log-sum-exp:
    lse = log sum_r exp(lse_r),   out = sum_r exp(lse_r - lse) * out_r
which equals one softmax over all entries (a rank with no entries has
lse_r = -inf and weight 0).

The pieces follow the same definitions as the single-rank oracle: the
indexer scores and Top-K rule (Model techniques map, "Indexer-selected sparse
attention" row) and the MLA attention over selected plus window entries.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np

from .attention import attend


def shard_bounds(T: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous [t0, t1) position ranges, sizes differing by at most one."""
    base, extra = divmod(T, world)
    out, t0 = [], 0
    for r in range(world):
        t1 = t0 + base + (1 if r < extra else 0)
        out.append((t0, t1))
        t0 = t1
    return out


def local_topk(scores_shard: np.ndarray, t0: int, K: int) -> Tuple[np.ndarray, np.ndarray]:
    """The shard's best min(K, n) entries as (scores float64, global positions
    int64), ranked by score descending then position ascending."""
    s = np.asarray(scores_shard, dtype=np.float64)
    pos = t0 + np.arange(s.shape[0], dtype=np.int64)
    order = np.lexsort((pos, -s))[:min(K, s.shape[0])]
    return s[order], pos[order]


def merge_topk(parts: Sequence[Tuple[np.ndarray, np.ndarray]], K: int) -> np.ndarray:
    """Global Top-K from every rank's local Top-K: int32 [K], ascending, -1 padded."""
    s = np.concatenate([p[0] for p in parts]) if parts else np.zeros(0)
    pos = np.concatenate([p[1] for p in parts]) if parts else np.zeros(0, np.int64)
    order = np.lexsort((pos, -s))[:min(K, s.shape[0])]
    take = np.sort(pos[order])
    out = np.full(K, -1, dtype=np.int32)
    out[:take.size] = take
    return out


def partial_attention(q: np.ndarray, X_shard: np.ndarray, scale: float):
    """One rank's (out [H, D], lse [H]) over its own entries (no sink: a sink is
    one extra denominator term, added once after the combine)."""
    return attend(q, X_shard, scale, None)


def combine(parts: Sequence[Tuple[np.ndarray, np.ndarray]], sink: np.ndarray | None = None):
    """Log-sum-exp merge of per-rank (out, lse), plus an optional sink logit."""
    lses = np.stack([p[1] for p in parts])                       # [R, H]
    outs = np.stack([p[0] for p in parts])                       # [R, H, D]
    m = lses.max(axis=0)
    if sink is not None:
        m = np.maximum(m, np.asarray(sink, dtype=np.float32).astype(np.float64))
    safe_m = np.where(np.isneginf(m), 0.0, m)
    wts = np.where(np.isneginf(lses), 0.0, np.exp(lses - safe_m[None, :]))   # [R, H]
    Z = wts.sum(axis=0)
    if sink is not None:
        Z = Z + np.exp(np.asarray(sink, dtype=np.float32).astype(np.float64) - safe_m)
    with np.errstate(invalid="ignore", divide="ignore"):
        out = np.where(Z[:, None] > 0, (wts[:, :, None] * outs).sum(axis=0) / Z[:, None], 0.0)
        lse = np.where(Z > 0, safe_m + np.log(Z), -np.inf)
    return out, lse
