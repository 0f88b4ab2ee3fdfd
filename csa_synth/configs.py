"""Workload shapes of the CSA2 sparse-attention step (synthetic, seeded).

Five workloads, from a tiny decode step to a 1M-token prefill chunk:

* ``tiny_decode``      - B1, 1 query, T=4096, 16 heads, indexer 4x64, K=256.
* ``decode_64k``       - B8, T=65536, 64 heads, indexer 8x64, K=2048, 1% outlier
                         channels x20 in the latents.
* ``stack_128k``       - B32, T=131072, three layers Full / Reindex / Reuse.
* ``hier_1m``          - B4, T=2^20, Full layer builds a 2048-block x 8-position
                         candidate pool, three Reindex layers score only the pool;
                         planted high-score keys every ~4096 positions.
* ``prefill_1m``       - 4096 causal queries whose last one sits at position
                         2^20 - 1 (prefix 1,044,480), bf16 latents.

All share latent width D=512 (448 nope + 64 rope, stored as one latent), indexer
head dim 64, window 128, softmax scale 1/sqrt(512).
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field
from typing import List, Optional

FULL, REINDEX, REUSE, SWA = 0, 1, 2, 3


@dataclass(frozen=True)
class LayerSpec:
    mode: int                 # FULL / REINDEX / REUSE
    owner: int                # layer whose main KV and indexer keys this layer reads
    reuse_from: int = -1      # REUSE: layer whose Top-K indices are reused
    build_pool: bool = False  # FULL: also build the hierarchical candidate pool
    pool_from: int = -1       # REINDEX: score only the pool built by this layer
    m: int = 1                # tokens per cache entry of the caches this layer owns (compressor ratio)


@dataclass(frozen=True)
class Config:
    name: str
    B: int
    T: int                    # cache length (positions 0..T-1), incl. the n_q new tokens
    H: int                    # attention query heads
    H_I: int                  # indexer heads
    K: int                    # Top-K
    seed: int
    layers: List[LayerSpec] = field(default_factory=lambda: [LayerSpec(FULL, 0)])
    n_q: int = 1              # query tokens per sequence (1 = decode)
    D: int = 512
    d_I: int = 64
    W: int = 128
    pool_blocks: int = 2048
    pool_block_len: int = 8
    outliers: bool = False    # 1% of latent channels x20
    outlier_gain: float = 20.0
    planted: bool = False     # planted high-score keys every ~4096 positions
    plant_stride: int = 4096
    bf16_latents: bool = False
    key_format: str = "e4m3"  # indexer keys: "e4m3" (plain cast) or "mxfp4" (E2M1 + E8M0 per 32)

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def n_win(self) -> int:
        """Window entries each query attends to."""
        return min(self.W, self.T)

    @property
    def win_rows(self) -> int:
        """Rows in a layer's window buffer: query t reads rows [t, t + n_win)."""
        return self.n_q + self.n_win - 1

    @property
    def owners(self) -> List[int]:
        """Layers whose main KV and indexer keys the stack reads (SWA layers read none)."""
        return sorted({l.owner for l in self.layers if l.mode != SWA})

    def ratio(self, owner: int) -> int:
        """Tokens per cache entry of an owner layer's main KV and indexer keys."""
        return self.layers[owner].m

    def entries(self, owner: int) -> int:
        """Completed cache entries of an owner layer (T tokens; a tail group waits)."""
        return self.T // self.ratio(owner)

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


def _ced_layers():
    L = [LayerSpec(SWA, 0), LayerSpec(SWA, 1)]
    for g in range(3):                                   # encoder groups, owners 2, 8, 14
        o = 2 + 6 * g
        L.append(LayerSpec(FULL, o, m=2))
        L += [LayerSpec(REUSE, o, reuse_from=o) for _ in range(5)]
    d = 20                                               # decoder owner
    L.append(LayerSpec(FULL, d, build_pool=True))
    L += [LayerSpec(REUSE, d, reuse_from=d) for _ in range(3)]
    for g in range(4):
        r = 24 + 4 * g
        L.append(LayerSpec(REINDEX, d, pool_from=d))
        L += [LayerSpec(REUSE, d, reuse_from=r) for _ in range(3)]
    return L


CONFIGS = {
    "tiny_decode": Config(name="tiny_decode", B=1, T=4096, H=16, H_I=4, K=256, seed=0),
    "decode_64k": Config(name="decode_64k", B=8, T=65536, H=64, H_I=8, K=2048, seed=1,
                         outliers=True),
    "stack_128k": Config(
        name="stack_128k", B=32, T=131072, H=64, H_I=8, K=2048, seed=2,
        layers=[LayerSpec(FULL, 0), LayerSpec(REINDEX, 0),
                LayerSpec(REUSE, 0, reuse_from=1)]),
    "hier_1m": Config(
        name="hier_1m", B=4, T=1 << 20, H=64, H_I=8, K=2048, seed=3, planted=True,
        layers=[LayerSpec(FULL, 0, build_pool=True),
                LayerSpec(REINDEX, 0, pool_from=0),
                LayerSpec(REINDEX, 0, pool_from=0),
                LayerSpec(REINDEX, 0, pool_from=0)]),
    "prefill_1m": Config(name="prefill_1m", B=1, T=1 << 20, H=64, H_I=8, K=2048, seed=4,
                         n_q=4096, bf16_latents=True),
    # the pages' own indexer shape and key format (32 heads x 128, MXFP4 keys
    # of 68 B, top-512): the oracle side of the next row of the scope table
    "decode_mx": Config(name="decode_mx", B=8, T=65536, H=64, H_I=32, K=512, seed=5, d_I=128,
                        key_format="mxfp4"),
    # the pages' 40-layer causal encoder-decoder stack: 2 SWA layers, the
    # encoder's 3 x [1 Full, 5 Reuse] over caches of one entry per 2 tokens,
    # the decoder's [1 Full (pool), 3 Reuse] then 4 x [1 Reindex in the pool,
    # 3 Reuse] over the decoder's own per-token caches
    "ced_40": Config(name="ced_40", B=4, T=1 << 17, H=64, H_I=8, K=2048, seed=6, layers=_ced_layers()),
    # a quarter-size prefill chunk (profiling captures that must stay small)
    "prefill_256k": Config(name="prefill_256k", B=1, T=1 << 18, H=64, H_I=8, K=2048, seed=4,
                           n_q=1024, bf16_latents=True),
}


def get_config(name: str, **overrides) -> Config:
    cfg = CONFIGS[name]
    return cfg.replace(**overrides) if overrides else cfg
