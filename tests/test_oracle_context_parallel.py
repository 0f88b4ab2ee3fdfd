"""Pins for the position-sharded decode (oracle/context_parallel.py), on CPU.

The sharded computation must equal the single-rank oracle: the merged Top-K
bit for bit, and the log-sum-exp combine to float64 rounding.  The last test
runs the exchange for real, as two gloo ranks on 127.0.0.1.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest

from oracle import context_parallel as cp
from oracle import indexer
from oracle.attention import attend

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_shard_bounds_cover_positions_once():
    for T in (1, 7, 100, 4097):
        for world in (1, 2, 3, 8):
            b = cp.shard_bounds(T, world)
            assert b[0][0] == 0 and b[-1][1] == T
            assert all(b[i][1] == b[i + 1][0] for i in range(world - 1))
            sizes = [t1 - t0 for t0, t1 in b]
            assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("T,K,world", [(1000, 64, 2), (1000, 64, 3), (50, 64, 4), (257, 100, 8), (12, 5, 5)])
def test_merged_topk_equals_global_topk_with_ties(T, K, world):
    rng = np.random.default_rng(T + K + world)
    scores = rng.integers(0, 20, T).astype(np.float64)          # heavy ties across shards
    parts = [cp.local_topk(scores[t0:t1], t0, K) for t0, t1 in cp.shard_bounds(T, world)]
    assert np.array_equal(cp.merge_topk(parts, K), indexer.topk(scores, K))


def test_mutation_merge_by_score_only_is_caught():
    """Dropping the position tie-break in the merge picks a different set."""
    T, K, world = 64, 8, 4
    scores = np.zeros(T)                                           # every score tied
    parts = [cp.local_topk(scores[t0:t1], t0, K) for t0, t1 in cp.shard_bounds(T, world)]
    s = np.concatenate([p[0] for p in parts])
    pos = np.concatenate([p[1] for p in parts])
    wrong = np.sort(pos[np.argsort(-s, kind="stable")[::-1][:K]])   # score order only, last ranks first
    assert not np.array_equal(wrong, indexer.topk(scores, K)[:K])


@pytest.mark.parametrize("sink", [False, True])
def test_combine_equals_one_softmax(sink):
    rng = np.random.default_rng(4 + sink)
    H, D, E = 8, 64, 300
    q = rng.standard_normal((H, D)).astype(np.float32)
    X = rng.standard_normal((E, D)) * 3
    s = rng.standard_normal(H).astype(np.float32) if sink else None
    ref_o, ref_l = attend(q, X, 0.125, s)
    cuts = [0, 0, 77, 78, 200, 300]                                 # includes empty ranks
    parts = [cp.partial_attention(q, X[a:b], 0.125) for a, b in zip(cuts[:-1], cuts[1:])]
    o, l = cp.combine(parts, s)
    assert np.allclose(o, ref_o, rtol=1e-12, atol=1e-13)
    assert np.allclose(l, ref_l, rtol=1e-12, atol=1e-13)


def test_combine_of_nothing_is_zero_and_neg_inf():
    H, D = 4, 16
    q = np.ones((H, D), np.float32)
    parts = [cp.partial_attention(q, np.zeros((0, D)), 0.1) for _ in range(3)]
    o, l = cp.combine(parts)
    assert np.all(o == 0) and np.all(np.isneginf(l))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _decode_rank(rank, world, port, out_dir):
    """One rank of a position-sharded decode of tiny_decode (T=3000, K=256)."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from csa_synth import get_config
    from oracle.case import SynthCase
    from oracle import quant
    from oracle import context_parallel as cpr
    from oracle import indexer as ix
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = get_config("tiny_decode", T=3000, K=256)
        case = SynthCase(cfg, 0)
        inp = case.inputs(0)
        t0, t1 = cpr.shard_bounds(cfg.T, world)[rank]
        keys = case.keys(0)[t0:t1]                                   # this rank's shard only
        S = ix.index_scores(inp.qI[0], inp.w[0], keys)
        local = cpr.local_topk(S, t0, cfg.K)
        gathered = [None] * world
        dist.all_gather_object(gathered, local)
        idx = cpr.merge_topk(gathered, cfg.K)
        mine = idx[(idx >= t0) & (idx < t1)].astype(np.int64)
        X = quant.fp4_dequant_rows(case.main_entries(0, mine)) if mine.size else np.zeros((0, cfg.D))
        if rank == world - 1:                                        # the newest positions hold the window
            X = np.concatenate([X, quant.fp8_window_dequant_rows(inp.window[0:cfg.n_win])])
        part = cpr.partial_attention(inp.q[0], X, cfg.softmax_scale)
        parts = [None] * world
        dist.all_gather_object(parts, part)
        if rank == 0:
            o, l = cpr.combine(parts)
            np.savez(os.path.join(out_dir, "sharded.npz"), idx=idx, out=o, lse=l)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_position_sharded_decode_gloo_world2(tmp_path):
    import torch.multiprocessing as mp
    from csa_synth import get_config
    from oracle.case import SynthCase
    mp.spawn(_decode_rank, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    got = np.load(tmp_path / "sharded.npz")
    cfg = get_config("tiny_decode", T=3000, K=256)
    ref = SynthCase(cfg, 0).run()[0]
    assert np.array_equal(got["idx"], ref.idx[0])
    assert np.allclose(got["out"], ref.out[0], rtol=1e-12, atol=1e-13)
    assert np.allclose(got["lse"], ref.lse[0], rtol=1e-12, atol=1e-13)
