"""Oracle-side encoding of the seeded synthetic workloads.

Takes the fp32 values drawn by ``csa_synth`` and encodes them with this
package's own quantisers, so that every stored byte the oracle compares
against is produced without the CUDA path.
"""
from __future__ import annotations

from functools import lru_cache

import numpy as np

from csa_synth import workload as wl
from csa_synth.configs import Config

from .quant import fp4_quant_rows, fp8_window_quant_rows, e4m3_cast
from .mxfp4 import mxfp4_quant_rows
from .compressor import compress
from .layers import LayerInputs, run_stack


class SynthCase:
    """Encoded inputs of one sequence ``b`` of a config (rows built on demand)."""

    def __init__(self, cfg: Config, b: int, sinks: bool = False, threads: int = 4,
                 dense_latents: bool = False):
        self.cfg = cfg
        self.b = b
        self.sinks = sinks
        self.threads = threads
        self.dense_latents = dense_latents   # hold all fp32 latents of an owner (large caches)
        self._keys = {}
        self._lat = {}

    def keys(self, owner: int) -> np.ndarray:
        """Encoded indexer keys of an owner's cache entries (entries pooled from
        m token rows by the compressor when the owner's ratio m > 1)."""
        if owner not in self._keys:
            c, m = self.cfg, self.cfg.ratio(owner)
            x = wl.index_key(c, owner, self.b, 0, c.entries(owner) * m, threads=self.threads)
            if m > 1:
                g = wl.index_gate(c, owner, self.b, 0, c.entries(owner) * m, threads=self.threads)
                x = compress(x.reshape(-1, m, c.d_I), g.reshape(-1, m, c.d_I)).astype(np.float32)
            self._keys[owner] = mxfp4_quant_rows(x) if c.key_format == "mxfp4" else e4m3_cast(x)
        return self._keys[owner]

    def _pooled_latents(self, owner: int, entries: np.ndarray) -> np.ndarray:
        c, m = self.cfg, self.cfg.ratio(owner)
        tok = (np.asarray(entries, dtype=np.int64)[:, None] * m + np.arange(m)).reshape(-1)
        x = wl.main_latent_at(c, owner, self.b, tok).reshape(-1, m, c.D)
        g = wl.main_gate_at(c, owner, self.b, tok).reshape(-1, m, c.D)
        return compress(x, g).astype(np.float32)

    def main_entries(self, owner: int, positions: np.ndarray) -> np.ndarray:
        if self.cfg.ratio(owner) > 1:
            return fp4_quant_rows(self._pooled_latents(owner, positions))
        if self.dense_latents:
            if owner not in self._lat:
                self._lat[owner] = wl.main_latent(self.cfg, owner, self.b, 0, self.cfg.T, threads=self.threads)
            return fp4_quant_rows(self._lat[owner][np.asarray(positions, dtype=np.int64)])
        return fp4_quant_rows(wl.main_latent_at(self.cfg, owner, self.b, positions))

    def main_range(self, owner: int, t0: int, n: int) -> np.ndarray:
        if self.cfg.ratio(owner) > 1:
            return self.main_entries(owner, np.arange(t0, t0 + n))
        return fp4_quant_rows(wl.main_latent(self.cfg, owner, self.b, t0, n, threads=self.threads))

    def inputs(self, layer: int) -> LayerInputs:
        c = self.cfg
        return LayerInputs(
            qI=e4m3_cast(wl.index_query(c, layer, self.b)),
            w=wl.index_weight(c, layer, self.b),
            q=wl.attn_query(c, layer, self.b),
            window=fp8_window_quant_rows(wl.window_latent(c, layer, self.b)),
            sink=wl.sink(c, layer) if self.sinks else None,
        )

    def run(self, queries=None, keep_scores=False):
        c = self.cfg
        return run_stack(c.layers, c.T, c.n_q, c.K, c.n_win, c.softmax_scale,
                         self.keys, self.main_entries, self.inputs, queries=queries,
                         pool_blocks=c.pool_blocks, pool_block_len=c.pool_block_len,
                         keep_scores=keep_scores, key_format=c.key_format, owner_len=c.entries)
