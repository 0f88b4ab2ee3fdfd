"""The m-token compressor of the encoder's CSA2 layers (oracle; test
infrastructure only).

DeepSeek-V4.1-Flash architecture database, cache groups: the encoder's main
KV (layers 2, 8, 14) and indexer K hold one shared K=V entry per 2 tokens
("tokens per entry" 2; completed entries are floor(context / 2), the
incomplete group's compressor state is excluded); the decoder's ratio-1
compressor "is a plain projection" with "nothing to pool, so no gate and no
fp32".  The projections themselves need trained weights and are outside the
step; what remains is the pooling of a group's m projected tokens.

Reading taken (the pages name a gate and fp32 but give no formula): per
channel d of a group of m tokens with values x[i, d] and gate logits
g[i, d],
    w[i, d] = exp(g[i, d]) / sum_j exp(g[j, d])        (softmax over the group)
    entry[d] = sum_i w[i, d] * x[i, d]
in floating point (float64 here; the kernel computes it in fp32).  m = 1 is
the plain case: entry = x, no gate.  The entry is then encoded like any
cache row (FP4 main KV, E4M3 indexer key).
"""
from __future__ import annotations

import numpy as np


def compress(x: np.ndarray, gate: np.ndarray | None = None) -> np.ndarray:
    """x [n, m, dim] (fp32 values), gate [n, m, dim] or None -> float64 [n, dim]."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    if x.shape[1] == 1:
        return x[:, 0].copy()
    g = np.asarray(gate, dtype=np.float32).astype(np.float64)
    g = g - g.max(axis=1, keepdims=True)        # the same softmax, overflow-free
    w = np.exp(g)
    w = w / w.sum(axis=1, keepdims=True)
    return (w * x).sum(axis=1)


def group_count(tokens: int, m: int) -> int:
    """Completed entries of a cache of `tokens` tokens (the tail group waits)."""
    return tokens // m
