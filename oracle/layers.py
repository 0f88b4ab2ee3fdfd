"""Full / Reindex / Reuse layer stacks of the CSA2 step (oracle).

Per the DeepSeek-V4.1 blog ("DeepSeek-V4.1-Flash", CSA2 paragraph) every
attention layer has one static mode: Full, Reindex or Reuse, sharing main KV
and indexer K across layers and reusing Top-K indices; in the decoder the
first Full layer builds a candidate pool that later indexing layers search.
The DeepSeek-V4.1-Flash architecture database (cross-layer cache fact) says
main KV and indexer K are owned by source layers that other CSA2 layers read,
and every layer keeps its own 128-token sliding-window KV.

Readings used here:
    Full    - scores all candidate positions with its own indexer queries and
              its owner's keys (itself), Top-K, optional pool; attends over its
              owner's main KV at the selected positions plus its own window.
    Reindex - its owner's keys and main KV, its own indexer queries/weights,
              a new Top-K (inside the pool when one is named), own window.
    Reuse   - the Top-K indices of the named earlier layer, its owner's main
              KV, its own window and attention queries; no scoring.
    SWA     - a sliding-window layer: attention over its own window alone
              (the stack's first two layers, architecture database layer
              pattern "2 SWA + 18 CSA2 m=2 + 20 CSA2 m=1").
An owner whose caches hold one entry per m tokens (the encoder's CSA2 m=2
layers) has owner_len(owner) = floor(T / m) entries, and its layers select
among those entries; windows stay per token.
Query t of a sequence with n_q new tokens and cache length T sits at position
T - n_q + t and sees positions [0, T - n_q + t] (decode: n_q = 1, all of
[0, T)); its window rows are [t, t + n_win) of the layer's window buffer.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Dict, List, Optional, Sequence

import numpy as np

from .indexer import index_scores, topk, build_pool
from .mxfp4 import mx_index_scores
from .attention import attend
from .quant import fp4_dequant_rows, fp8_window_dequant_rows

FULL, REINDEX, REUSE, SWA = 0, 1, 2, 3


@dataclass
class LayerInputs:
    """One layer's own tensors for one sequence (codes as stored)."""
    qI: np.ndarray                  # uint8 [n_q, H_I, d_I]
    w: np.ndarray                   # fp32 [n_q, H_I]
    q: np.ndarray                   # fp32 [n_q, H, D]
    window: np.ndarray              # uint8 [win_rows, 528]
    sink: Optional[np.ndarray] = None


@dataclass
class LayerResult:
    idx: np.ndarray                 # int32 [n_sel_queries, K]
    out: np.ndarray                 # float64 [n_sel_queries, H, D]
    lse: np.ndarray                 # float64 [n_sel_queries, H]
    pool: Optional[np.ndarray] = None
    pool_len: int = 0
    scores: Optional[List[np.ndarray]] = None


def run_stack(layers: Sequence, T: int, n_q: int, K: int, n_win: int, scale: float,
              keys: Callable[[int], np.ndarray],
              main_entries: Callable[[int, np.ndarray], np.ndarray],
              inputs: Callable[[int], LayerInputs],
              queries: Optional[Sequence[int]] = None,
              pool_blocks: int = 2048, pool_block_len: int = 8,
              keep_scores: bool = False, key_format: str = "e4m3",
              owner_len: Optional[Callable[[int], int]] = None) -> List[LayerResult]:
    """Run a layer stack for one sequence.

    ``layers``: objects with mode / owner / reuse_from / build_pool / pool_from.
    ``keys(owner)``: uint8 indexer keys of the owner layer: [T, d_I] E4M3 codes,
    or [T, d_I/2 + d_I/32] MXFP4 entries when ``key_format`` is "mxfp4".
    ``main_entries(owner, positions)``: uint8 [n, 288] main-KV entries.
    ``inputs(layer)``: that layer's LayerInputs.
    ``queries``: query token indices to evaluate (default all n_q).
    """
    qs = list(range(n_q)) if queries is None else list(queries)
    score = mx_index_scores if key_format == "mxfp4" else index_scores
    results: List[LayerResult] = []
    for li, L in enumerate(layers):
        inp = inputs(li)
        idx_rows, scores_rows = [], []
        pool, pool_len = None, 0
        T_o = T if owner_len is None or L.mode == SWA else owner_len(L.owner)
        if T_o != T:
            assert n_q == 1, "compressed caches are read at decode"
        if L.mode == SWA:
            idx_rows = [np.full(K, -1, dtype=np.int32) for _ in qs]
        elif L.mode == REUSE:
            src = results[L.reuse_from]
            idx_rows = list(src.idx)
        else:
            kc = keys(L.owner)
            for t in qs:
                n_t = T_o - n_q + t + 1
                if L.mode == REINDEX and L.pool_from >= 0:
                    P = results[L.pool_from]
                    ppos = P.pool[:P.pool_len].astype(np.int64)
                    S = score(inp.qI[t], inp.w[t], kc[ppos])
                    idx_rows.append(topk(S, K, ppos))
                else:
                    S = score(inp.qI[t], inp.w[t], kc[:n_t])
                    idx_rows.append(topk(S, K))
                    if L.build_pool:
                        pool, pool_len = build_pool(S, pool_blocks, pool_block_len)
                if keep_scores:
                    scores_rows.append(S)
        outs, lses = [], []
        for r, t in enumerate(qs):
            sel = idx_rows[r]
            sel = sel[sel >= 0].astype(np.int64)
            Xm = fp4_dequant_rows(main_entries(L.owner, sel)) if sel.size else np.zeros((0, 512))
            Xw = fp8_window_dequant_rows(inp.window[t:t + n_win])
            o, l = attend(inp.q[t], np.concatenate([Xm, Xw], axis=0), scale, inp.sink)
            outs.append(o)
            lses.append(l)
        results.append(LayerResult(idx=np.stack(idx_rows).astype(np.int32), out=np.stack(outs),
                                   lse=np.stack(lses), pool=pool, pool_len=pool_len,
                                   scores=scores_rows if keep_scores else None))
    return results
