"""Device-resident workloads for the CUDA path (GPU tests and the benchmark).

The fp32 / bf16 values come from ``csa_synth.workload`` (seeded, chunked);
they are uploaded and encoded ON THE DEVICE by the library under test
(``csa_quant_kv``), exactly as a caller would fill its caches.  The oracle
never imports this module: it encodes the same values with its own code.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

from . import workload as wl
from .configs import Config, FULL, REINDEX, REUSE, SWA

UPLOAD_ROWS = 1 << 16


def _lib():
    import indexer_selected_sparse_csa2_b200 as csa
    return csa


@dataclass
class DeviceLayer:
    qI: object                      # uint8 [B, n_q, H_I, 64]
    w: object                       # fp32 [B, n_q, H_I]
    q: object                       # fp32 [B, n_q, H, 512]
    win: object                     # uint8 [B, win_rows, 528]
    idx: object                     # int32 [B, n_q, K]
    out: object                     # fp32 [B, n_q, H, 512]
    lse: object                     # fp32 [B, n_q, H]
    sink: Optional[object] = None
    pool: Optional[object] = None   # int32 [B, pool_blocks * pool_block_len]
    pool_len: Optional[object] = None
    scores: Optional[object] = None


class DeviceCase:
    """All caches and per-layer tensors of one config on ``device``."""

    def __init__(self, cfg: Config, device: str = "cuda", sinks: bool = False, threads: int = 8,
                 keep_scores: bool = False, batches: Optional[List[int]] = None):
        import torch
        csa = _lib()
        if cfg.key_format not in ("e4m3", "mxfp4"):
            raise NotImplementedError(f"indexer key format {cfg.key_format!r} has no device encoder")
        self.cfg = cfg
        self.device = device
        B, T = cfg.B, cfg.T
        self.keys: Dict[int, object] = {}
        self.key_scales: Dict[int, object] = {}     # MXFP4 keys: exponent bytes [B, T, d_I / 32]
        self.kv: Dict[int, object] = {}
        mx = cfg.key_format == "mxfp4"
        for o in cfg.owners:
            E, m = cfg.entries(o), cfg.ratio(o)
            keys = torch.empty((B, E, cfg.d_I // 2 if mx else cfg.d_I), dtype=torch.uint8, device=device)
            if mx:
                self.key_scales[o] = torch.empty((B, E, cfg.d_I // 32), dtype=torch.uint8, device=device)
            kv = torch.empty((B, E, csa.FP4_ENTRY_BYTES), dtype=torch.uint8, device=device)
            for b in range(B):
                for e0 in range(0, E, UPLOAD_ROWS):
                    n = min(UPLOAD_ROWS, E - e0)
                    kx = torch.from_numpy(wl.index_key(cfg, o, b, e0 * m, n * m, threads=threads)).to(device)
                    lx = self._latent_tensor(wl.main_latent(cfg, o, b, e0 * m, n * m, threads=threads))
                    if m == 1:
                        if o in self.key_scales:
                            csa.csa_quant_mxfp4(kx, keys[b, e0:e0 + n], self.key_scales[o][b, e0:e0 + n])
                        else:
                            csa.csa_quant_kv(kx, csa.CSA_FMT_FP8_E4M3_PLAIN, keys[b, e0:e0 + n])
                        csa.csa_quant_kv(lx, csa.CSA_FMT_FP4_E2M1_E4M3X16, kv[b, e0:e0 + n])
                    else:
                        # the compressor pools each group of m token rows into one entry
                        kg = torch.from_numpy(wl.index_gate(cfg, o, b, e0 * m, n * m, threads=threads)).to(device)
                        mg = torch.from_numpy(wl.main_gate(cfg, o, b, e0 * m, n * m, threads=threads)).to(device)
                        csa.csa_compress_kv(kx, kg, m, csa.CSA_FMT_FP8_E4M3_PLAIN, keys[b, e0:e0 + n])
                        csa.csa_compress_kv(lx, mg, m, csa.CSA_FMT_FP4_E2M1_E4M3X16, kv[b, e0:e0 + n])
            self.keys[o] = keys
            self.kv[o] = kv
        self.layers: List[DeviceLayer] = []
        for li, L in enumerate(cfg.layers):
            qI_f = np.stack([wl.index_query(cfg, li, b) for b in range(B)])         # [B, n_q, H_I, 64]
            qI = torch.empty(qI_f.shape, dtype=torch.uint8, device=device)
            qf = torch.from_numpy(qI_f.reshape(-1, cfg.d_I)).to(device)
            csa.csa_quant_kv(qf, csa.CSA_FMT_FP8_E4M3_PLAIN, qI.view(-1, cfg.d_I))
            w = torch.from_numpy(np.stack([wl.index_weight(cfg, li, b) for b in range(B)])).to(device)
            q = torch.from_numpy(np.stack([wl.attn_query(cfg, li, b) for b in range(B)])).to(device)
            win = torch.empty((B, cfg.win_rows, csa.FP8_ENTRY_BYTES), dtype=torch.uint8, device=device)
            for b in range(B):
                wx = self._latent_tensor(wl.window_latent(cfg, li, b))
                csa.csa_quant_kv(wx, csa.CSA_FMT_FP8_E4M3_UE8M0X32, win[b])
            dl = DeviceLayer(
                qI=qI, w=w.contiguous(), q=q.contiguous(), win=win,
                idx=torch.full((B, cfg.n_q, cfg.K), -7, dtype=torch.int32, device=device),
                out=torch.zeros((B, cfg.n_q, cfg.H, cfg.D), dtype=torch.float32, device=device),
                lse=torch.zeros((B, cfg.n_q, cfg.H), dtype=torch.float32, device=device),
            )
            if sinks:
                dl.sink = torch.from_numpy(wl.sink(cfg, li)).to(device)
            if L.build_pool:
                dl.pool = torch.full((B, cfg.pool_blocks * cfg.pool_block_len), -7, dtype=torch.int32,
                                     device=device)
                dl.pool_len = torch.zeros(B, dtype=torch.int32, device=device)
            if keep_scores and L.mode in (FULL, REINDEX):
                n = cfg.entries(L.owner)
                if L.mode == REINDEX and L.pool_from >= 0:
                    n = cfg.pool_blocks * cfg.pool_block_len
                dl.scores = torch.zeros((B, n), dtype=torch.float32, device=device)
            self.layers.append(dl)

    def _latent_tensor(self, x: np.ndarray):
        import torch
        t = torch.from_numpy(x).to(self.device)
        return t.to(torch.bfloat16) if self.cfg.bf16_latents else t

    # ------------------------------------------------------------------
    def _put(self, arena, t):
        """Copy ``t`` into the next 256-byte-aligned slot of ``arena`` (a dict
        holding a uint8 device buffer and a cursor) and return the view."""
        n = t.numel() * t.element_size()
        off = (arena["off"] + 255) // 256 * 256
        if off + n > arena["buf"].numel():
            raise ValueError("step I/O arena too small")
        v = arena["buf"][off:off + n].view(t.dtype).view(t.shape)
        v.copy_(t)
        arena["off"] = off + n
        return v

    def layer_descs(self, append_rows: bool = False, packed: bool = False):
        """ctypes LayerDesc array for the config's stack.  With ``append_rows``
        every owner layer re-encodes the newest token (position T-1) of its
        main KV and indexer key, and every layer its newest window row, as part
        of the step (values from the seeded generator).  With ``packed`` the
        step's per-token inputs are moved into two contiguous device buffers,
        ``self.step_q`` (every layer's attention query) and ``self.step_in``
        (index queries, head weights, appended source rows), and its outputs
        (out, lse, idx of every layer, layer by layer) into ``self.step_out``
        with layer i at bytes ``self.step_out_ranges[i]``, so that a caller
        moves each with one host <-> device copy (per layer for the outputs)."""
        import torch
        csa = _lib()
        cfg = self.cfg
        descs = []
        self._append_src = []
        src_arena = None
        if packed:
            per_tok = 4 * (2 * 512 + cfg.d_I) * max(cfg.n_q, 1)
            n_in = sum(dl.q.numel() * 4 + dl.qI.numel() + dl.w.numel() * 4 + 1024 for dl in self.layers)
            n_in += len(cfg.layers) * (cfg.B * per_tok + 1024)
            src_arena = {"buf": torch.empty(n_in, dtype=torch.uint8, device=self.device), "off": 0}
            n_q = sum(dl.q.numel() * 4 + 256 for dl in self.layers)
            q_arena = {"buf": torch.empty(n_q, dtype=torch.uint8, device=self.device), "off": 0}
            n_out = sum(dl.out.numel() * 4 + dl.lse.numel() * 4 + dl.idx.numel() * 4 + 1024 for dl in self.layers)
            out_arena = {"buf": torch.empty(n_out, dtype=torch.uint8, device=self.device), "off": 0}
            self.step_out_ranges = []
            for dl in self.layers:
                dl.q = self._put(q_arena, dl.q)
                dl.qI, dl.w = (self._put(src_arena, t) for t in (dl.qI, dl.w))
                o0 = (out_arena["off"] + 255) // 256 * 256
                dl.out, dl.lse, dl.idx = (self._put(out_arena, t) for t in (dl.out, dl.lse, dl.idx))
                self.step_out_ranges.append((o0, out_arena["off"]))
        put = (lambda t: self._put(src_arena, t)) if packed else (lambda t: t)
        for li, L in enumerate(cfg.layers):
            d = csa.LayerDesc()
            d.mode = L.mode
            d.reuse_from = L.reuse_from
            d.pool_from = L.pool_from
            dl = self.layers[li]
            o = L.owner
            if append_rows:
                # the step's new tokens: position T-1 of every sequence at decode
                # (rows strided by the batch stride), positions [T-n_q, T) of the
                # single sequence of a prefill chunk
                n_new = cfg.n_q
                if n_new > 1 and cfg.B != 1:
                    raise ValueError("prefill appends are built for one sequence")
                jobs = []
                t_new = cfg.T - n_new
                if o == li and L.mode != SWA and cfg.ratio(o) == 1:
                    # (an owner with m > 1 gains an entry only when a group of m
                    # tokens completes; its caches are built whole above)
                    if n_new == 1:
                        mx = torch.stack([self._latent_tensor(wl.main_latent(cfg, o, b, cfg.T - 1, 1))[0]
                                          for b in range(cfg.B)])
                        kx = torch.from_numpy(np.stack([wl.index_key(cfg, o, b, cfg.T - 1, 1)[0]
                                                        for b in range(cfg.B)])).to(self.device)
                        kvrow, krow = self.kv[o][:, cfg.T - 1], self.keys[o][:, cfg.T - 1]
                        kv_stride, k_stride = self.kv[o].stride(0), self.keys[o].stride(0)
                    else:
                        mx = self._latent_tensor(wl.main_latent(cfg, o, 0, t_new, n_new))
                        kx = torch.from_numpy(wl.index_key(cfg, o, 0, t_new, n_new)).to(self.device)
                        kvrow, krow = self.kv[o][0, t_new:], self.keys[o][0, t_new:]
                        kv_stride, k_stride = self.kv[o].stride(1), self.keys[o].stride(1)
                    mx = put(mx)
                    if cfg.key_format == "e4m3":
                        kx = put(kx)
                    jobs.append(csa.quant_job(mx, csa.CSA_FMT_FP4_E2M1_E4M3X16, kvrow, kv_stride))
                    if cfg.key_format == "e4m3":       # (MXFP4 keys are encoded whole above)
                        jobs.append(csa.quant_job(kx, csa.CSA_FMT_FP8_E4M3_PLAIN, krow, k_stride))
                    self._append_src += [mx, kx]
                r0 = cfg.win_rows - n_new
                if n_new == 1:
                    wx = torch.stack([self._latent_tensor(wl.window_latent(cfg, li, b))[r0]
                                      for b in range(cfg.B)])
                    wrow, w_stride = dl.win[:, r0], dl.win.stride(0)
                else:
                    wx = self._latent_tensor(wl.window_latent(cfg, li, 0)[r0:])
                    wrow, w_stride = dl.win[0, r0:], dl.win.stride(1)
                wx = put(wx)
                jobs.append(csa.quant_job(wx, csa.CSA_FMT_FP8_E4M3_UE8M0X32, wrow, w_stride))
                self._append_src.append(wx)
                for k, j in enumerate(jobs):
                    d.append[k] = j
            if L.mode in (FULL, REINDEX):
                d.index = csa.index_args(
                    keys=self.keys[o], key_scales=self.key_scales.get(o), q=dl.qI, w=dl.w, K=cfg.K, idx=dl.idx,
                    T=cfg.entries(o), n_q=cfg.n_q,
                    pool_out=dl.pool, pool_out_len=dl.pool_len, pool_blocks=cfg.pool_blocks,
                    pool_block_len=cfg.pool_block_len, scores=dl.scores)
            d.attn = csa.attn_args(q=dl.q, kv=self.kv[o] if L.mode != SWA else None, idx=None, win=dl.win,
                                   n_win=cfg.n_win, softmax_scale=cfg.softmax_scale, out=dl.out, lse=dl.lse,
                                   sink=dl.sink, K=0)
            d._keep = (getattr(d, "_keep", None), self.keys, self.kv, dl)
            descs.append(d)
        if packed:
            self.step_in = src_arena["buf"][:src_arena["off"]]
            self.step_q = q_arena["buf"][:q_arena["off"]]
            self.step_out = out_arena["buf"][:out_arena["off"]]
        return csa.make_layer_array(descs)
