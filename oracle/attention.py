"""Sparse MLA attention over selected FP4 entries plus the FP8 window (oracle).

Per the Model techniques map (DeepSeek-V4.1-Flash): the attention is
multi-head latent attention with a single latent KV head ("Multi-head latent
attention" and "Grouped-query attention" rows: num_key_value_heads = 1 is the
MLA latent); every layer keeps a 128-token sliding-window KV ("Sliding-window
attention" row); each query attends only to the indexer's selected entries
("Indexer-selected sparse attention" row); an optional learned per-head sink
logit joins the softmax denominator ("Learnable attention sink" row, initial
value -inf).  The architecture database (cache groups) stores one shared K=V
entry of 512 elements, so keys and values are the same dequantised latent,
all 512 dimensions (448 nope + 64 rope; the rope part is already rotated
before caching, "Post-RoPE KV-cache quantization" in the techniques map).

For query head h of one token, over entries x_e (the valid selected rows then
the window rows, duplicates kept):
    l_e   = scale * <q_h, x_e>
    m     = max(max_e l_e, sink_h)              (sink term only when given)
    Z     = sum_e exp(l_e - m) + exp(sink_h - m)
    out_h = sum_e exp(l_e - m) * x_e / Z
    lse_h = m + log Z                           (natural log)
All in float64.  With no entries and no sink: out = 0, lse = -inf.
"""
from __future__ import annotations

import numpy as np


def attend(q: np.ndarray, X: np.ndarray, scale: float, sink: np.ndarray | None = None):
    """q [H, D] (fp32 values), X [E, D] float64 entries -> (out [H, D], lse [H]) float64."""
    q = np.asarray(q, dtype=np.float32).astype(np.float64)
    X = np.asarray(X, dtype=np.float64)
    H = q.shape[0]
    sc = float(np.float32(scale))
    if X.shape[0] == 0 and sink is None:
        return np.zeros((H, X.shape[1] if X.ndim == 2 else q.shape[1])), np.full(H, -np.inf)
    logits = (q @ X.T) * sc                                     # [H, E]
    m = logits.max(axis=1) if X.shape[0] else np.full(H, -np.inf)
    if sink is not None:
        s = np.asarray(sink, dtype=np.float32).astype(np.float64)
        m = np.maximum(m, s)
    p = np.exp(logits - m[:, None])
    Z = p.sum(axis=1)
    if sink is not None:
        Z = Z + np.exp(s - m)
    out = (p @ X) / Z[:, None]
    return out, m + np.log(Z)
