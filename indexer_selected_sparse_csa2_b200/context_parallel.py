"""Context-parallel decode of one long sequence: host orchestration.

The cache positions [0, T) are split into contiguous shards, one per rank
(``shard_bounds``); rank r holds its shard's indexer keys and main KV, and
the last rank (the newest positions) also holds the sliding window.  One
decode step of one layer is two exchange rounds:

1. every rank scores its shard and keeps its local Top-K as (score, global
   position) pairs; the pairs are all-gathered and every rank merges them
   into the global Top-K (``csa_cp_merge_topk``: the K best of the union by
   score, then lower position; exact, since every global winner is among the
   K best of its own shard);
2. every rank attends over the selected entries it owns (plus the window on
   the last rank) and returns (out_r, lse_r); these are all-gathered and
   combined by log-sum-exp (``csa_cp_combine``), which equals one softmax
   over all the entries.

The arithmetic runs in the library's kernels; this module only sequences the
calls and the exchange.  ``cp_decode`` takes the per-rank operations and the
communicator as arguments, so the same sequencing runs with the device
kernels over NCCL (``DeviceShard`` + ``TorchComm``) or, in tests, with other
implementations of the same operations.
"""
from __future__ import annotations

import math
from typing import List, Tuple


def shard_bounds(T: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous [t0, t1) shards of [0, T) in rank order, sizes differing by at most one."""
    base, extra = divmod(T, world)
    out, t0 = [], 0
    for r in range(world):
        t1 = t0 + base + (1 if r < extra else 0)
        out.append((t0, t1))
        t0 = t1
    return out


class TorchComm:
    """All-gather over a torch.distributed process group (NCCL for device
    tensors, gloo for host tensors): returns the ranks' tensors stacked in
    rank order."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def all_gather(self, t):
        import torch
        parts = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(parts, t.contiguous(), group=self.group)
        return torch.stack(parts)


def cp_decode(ops, comm, rank: int, world: int, T: int):
    """One decode step of one layer on this rank.  ``ops`` provides
    local_topk(t0, t1) -> (pair_score, pair_pos), merge(scores [R..],
    positions [R..]) -> idx, attend(idx, t0, t1, with_window) -> (out, lse)
    and combine(outs [R..], lses [R..]) -> (out, lse).  Every rank takes the
    same collective steps in the same order.  Returns (idx, out, lse)."""
    t0, t1 = shard_bounds(T, world)[rank]
    pair_score, pair_pos = ops.local_topk(t0, t1)
    idx = ops.merge(comm.all_gather(pair_score), comm.all_gather(pair_pos))
    out_r, lse_r = ops.attend(idx, t0, t1, rank == world - 1)
    out, lse = ops.combine(comm.all_gather(out_r), comm.all_gather(lse_r))
    return idx, out, lse


class DeviceShard:
    """The per-rank operations on this GPU's shard with the library's kernels.

    keys [B, T_shard, 64] E4M3 and kv [B, T_shard, 288] hold positions
    [t0, t1); q fp32 [B, 1, H, 512], qI E4M3 [B, 1, H_I, 64], w fp32
    [B, 1, H_I]; win [B, rows, 528] (used on the last rank only)."""

    def __init__(self, keys, kv, q, qI, w, win, n_win: int, K: int, softmax_scale: float, sink=None):
        self.keys, self.kv, self.q, self.qI, self.w, self.win = keys, kv, q, qI, w, win
        self.n_win, self.K, self.scale, self.sink = n_win, K, softmax_scale, sink

    def local_topk(self, t0: int, t1: int):
        import torch
        from . import index_args, csa_index_topk, csa_cp_local_pairs
        B, Ts = self.keys.shape[0], self.keys.shape[1]
        dev = self.keys.device
        idx = torch.full((B, 1, self.K), -1, dtype=torch.int32, device=dev)
        sc = torch.empty((B, max(Ts, 1)), dtype=torch.float32, device=dev)
        ps = torch.empty((B, self.K), dtype=torch.float32, device=dev)
        pp = torch.empty((B, self.K), dtype=torch.int32, device=dev)
        if Ts > 0:
            csa_index_topk(index_args(keys=self.keys, q=self.qI, w=self.w, K=self.K, idx=idx, scores=sc),
                           device=dev)
        csa_cp_local_pairs(idx.view(B, self.K), sc, t0, ps, pp)
        return ps, pp

    def merge(self, gathered_score, gathered_pos):
        import torch
        from . import csa_cp_merge_topk
        B = gathered_score.shape[1]
        idx = torch.empty((B, self.K), dtype=torch.int32, device=gathered_score.device)
        csa_cp_merge_topk(gathered_score, gathered_pos, self.K, idx)
        return idx

    def attend(self, idx, t0: int, t1: int, with_window: bool):
        import torch
        from . import attn_args, csa_sparse_attn, csa_cp_localize
        B, H = self.q.shape[0], self.q.shape[2]
        dev = self.q.device
        local = torch.empty_like(idx)
        csa_cp_localize(idx, t0, t1, local)
        out = torch.empty((B, 1, H, 512), dtype=torch.float32, device=dev)
        lse = torch.empty((B, 1, H), dtype=torch.float32, device=dev)
        n_win = self.n_win if with_window else 0
        a = attn_args(q=self.q, kv=self.kv, idx=local.view(B, 1, self.K), win=self.win if n_win else None,
                      n_win=n_win, softmax_scale=self.scale, out=out, lse=lse, K=self.K)
        csa_sparse_attn(a, device=dev)
        return out.view(B, H, 512), lse.view(B, H)

    def combine(self, outs, lses):
        import torch
        from . import csa_cp_combine
        R, B, H = lses.shape
        out = torch.empty((B, H, 512), dtype=torch.float32, device=outs.device)
        lse = torch.empty((B, H), dtype=torch.float32, device=outs.device)
        csa_cp_combine(outs.contiguous(), lses.contiguous(), out, lse, sink=self.sink)
        return out, lse
