"""Lightning-indexer scores, Top-K and the hierarchical candidate pool (oracle).

Scores (a3).  The pages give the indexer's role and shapes (Model techniques
map, "Indexer-selected sparse attention (DeepSeek Sparse Attention)" row: an
indexer with its own heads scores past tokens and each query attends only to
the index_topk selected ones).  The score of cached position s for one query is
    S[s] = sum_j w[j] * max(0, sum_d qI[j, d] * kI[s, d])
with qI, kI stored as E4M3 codes and w fp32.  The dot products are computed
exactly in int64 (every E4M3 value is an integer multiple of 2^-9, so
dot * 2^18 is an integer of magnitude below 2^42); the weighted head sum is
taken in float64, heads in ascending order.

Top-K (a4).  The K largest scores; equal scores are broken towards the lower
position; if fewer than K candidates exist all of them are returned.  Output
is the selected positions in ascending order, padded with -1 to length K.

Pool (a5).  DeepSeek-V4.1-Flash architecture database, token-selection fact:
the decoder's hierarchical indexer is limited to "a 2048-block x 8-position
candidate pool"; the DeepSeek-V4.1 blog (CSA2 paragraph) says the pool is built
by the first Full-mode layer and later indexing layers search only inside it;
the Model techniques map lists "Blockwise candidate-pool selection for sparse
indexing".  Reading taken here: positions are grouped into aligned blocks
[8i, 8i+8) (the last block clipped at the cache length); a block's score is the
maximum score of its positions; the pool is the positions of the top 2048
blocks (ties towards the lower block), ascending, padded with -1.

Reindex over the pool (a6): the scores of the pool positions only (same keys,
this layer's queries and weights), then Top-K among them; ties resolve to the
lower position because the pool is ascending.
"""
from __future__ import annotations

import numpy as np

from .codecs import e4m3_int


def head_dots(q_codes: np.ndarray, k_codes: np.ndarray) -> np.ndarray:
    """Exact int64 dot products * 2^18: q [H_I, d], k [n, d] codes -> [n, H_I]."""
    qi = e4m3_int(q_codes)
    ki = e4m3_int(k_codes)
    out = np.empty((ki.shape[0], qi.shape[0]), dtype=np.int64)
    step = 1 << 16
    for s in range(0, ki.shape[0], step):
        out[s:s + step] = ki[s:s + step] @ qi.T
    return out


def index_scores(q_codes: np.ndarray, w: np.ndarray, k_codes: np.ndarray) -> np.ndarray:
    """float64 [n] scores of n keys for one query (q_codes [H_I, d], w [H_I])."""
    dots = head_dots(q_codes, k_codes).astype(np.float64) * np.ldexp(1.0, -18)   # exact
    wj = np.asarray(w, dtype=np.float32).astype(np.float64)
    S = np.zeros(dots.shape[0], dtype=np.float64)
    for j in range(wj.shape[0]):
        S += wj[j] * np.maximum(dots[:, j], 0.0)
    return S


def topk(scores: np.ndarray, K: int, positions: np.ndarray | None = None) -> np.ndarray:
    """int32 [K]: positions of the K largest scores (ties -> lower position), ascending, -1 padded."""
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.shape[0]
    pos = np.arange(n, dtype=np.int64) if positions is None else np.asarray(positions, dtype=np.int64)
    order = np.lexsort((pos, -scores))          # by score descending, then position ascending
    take = np.sort(pos[order[:min(K, n)]])
    out = np.full(K, -1, dtype=np.int32)
    out[:take.size] = take
    return out


def block_max(scores: np.ndarray, block_len: int) -> np.ndarray:
    """Max score of each aligned block [block_len*i, block_len*(i+1)), last block clipped."""
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.shape[0]
    nb = -(-n // block_len)
    padded = np.full(nb * block_len, -np.inf)
    padded[:n] = scores
    return padded.reshape(nb, block_len).max(axis=1)


def build_pool(scores: np.ndarray, pool_blocks: int, block_len: int):
    """(pool int32 [pool_blocks*block_len] ascending / -1 padded, valid count)."""
    n = scores.shape[0]
    blocks = topk(block_max(scores, block_len), pool_blocks)
    blocks = blocks[blocks >= 0].astype(np.int64)
    pos = (blocks[:, None] * block_len + np.arange(block_len)[None, :]).reshape(-1)
    pos = pos[pos < n]
    pool = np.full(pool_blocks * block_len, -1, dtype=np.int32)
    pool[:pos.size] = pos
    return pool, int(pos.size)


def reindex_topk(q_codes, w, k_codes_all: np.ndarray, pool: np.ndarray, pool_len: int, K: int):
    """Top-K restricted to pool positions; returns (idx int32 [K], pool scores)."""
    ppos = np.asarray(pool[:pool_len], dtype=np.int64)
    S = index_scores(q_codes, w, k_codes_all[ppos])
    return topk(S, K, ppos), S
