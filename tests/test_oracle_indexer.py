"""Pins for the oracle's indexer scores, Top-K and candidate pool (CPU only)."""
from fractions import Fraction

import numpy as np
import pytest

from oracle import indexer, codecs, quant
from csa_synth import get_config
from csa_synth import workload as wl


def _frac_scores(qc, w, kc):
    """Scores by exact rational arithmetic, plain Python loops."""
    out = []
    for s in range(kc.shape[0]):
        tot = Fraction(0)
        for j in range(qc.shape[0]):
            dot = Fraction(0)
            for d in range(qc.shape[1]):
                dot += Fraction(float(codecs.e4m3_decode(qc[j, d]))) * Fraction(float(codecs.e4m3_decode(kc[s, d])))
            tot += Fraction(float(np.float32(w[j]))) * max(dot, Fraction(0))
        out.append(tot)
    return out


def check_scores(score_fn):
    rng = np.random.default_rng(21)
    qc = quant.e4m3_cast(rng.standard_normal((3, 16)).astype(np.float32) * 4)
    kc = quant.e4m3_cast(rng.standard_normal((40, 16)).astype(np.float32) * 4)
    kc[5] = 0x7E          # saturated keys, extreme products
    qc[0, :] = 0x7E
    w = rng.random(3).astype(np.float32)
    w[1] = 0.0
    exact = _frac_scores(qc, w, kc)
    got = score_fn(qc, w, kc)
    return all(abs(Fraction(float(g)) - e) <= abs(e) * Fraction(1, 2 ** 50) for g, e in zip(got, exact))


def test_scores_vs_exact_rational_bruteforce():
    assert check_scores(indexer.index_scores)


def test_scores_mutation_no_relu_is_caught():
    def no_relu(qc, w, kc):
        d = indexer.head_dots(qc, kc) * 2.0 ** -18
        return (d * w[None, :].astype(np.float64)).sum(axis=1)
    assert not check_scores(no_relu)


def test_int64_dots_equal_float64_blas():
    rng = np.random.default_rng(22)
    qc = quant.e4m3_cast(rng.standard_normal((8, 64)).astype(np.float32) * 50)
    kc = quant.e4m3_cast(rng.standard_normal((5000, 64)).astype(np.float32) * 50)
    a = indexer.head_dots(qc, kc).astype(np.float64) * 2.0 ** -18
    b = codecs.e4m3_decode(kc) @ codecs.e4m3_decode(qc).T     # exact: < 2^24 with 2^-18 grain
    assert np.array_equal(a, b)


def check_topk(topk_fn):
    rng = np.random.default_rng(23)
    for n in [1, 2, 7, 31, 64, 257, 300]:
        for K in [1, 5, 64, 256, 400]:
            s = rng.integers(0, 6, size=n).astype(np.float64)      # many forced ties
            got = topk_fn(s, K)
            ranked = sorted(range(n), key=lambda i: (-s[i], i))[:min(K, n)]
            exp = sorted(ranked) + [-1] * (K - min(K, n))
            if list(got) != exp:
                return False
    return True


def test_topk_vs_full_sort_with_ties():
    assert check_topk(indexer.topk)


def test_topk_mutation_highest_index_tiebreak_is_caught():
    def bad(s, K):
        n = len(s)
        order = np.lexsort((-np.arange(n), -np.asarray(s)))
        take = np.sort(order[:min(K, n)])
        out = np.full(K, -1, np.int32)
        out[:take.size] = take
        return out
    assert not check_topk(bad)


def test_topk_negative_zero_ties():
    s = np.array([0.0, -0.0, 0.0, -0.0])
    assert list(indexer.topk(s, 2)) == [0, 1]


def test_pool_equals_all_when_pool_covers_everything():
    rng = np.random.default_rng(24)
    s = rng.random(100)
    pool, n = indexer.build_pool(s, pool_blocks=20, block_len=8)   # 13 blocks < 20
    assert n == 100 and list(pool[:100]) == list(range(100)) and np.all(pool[100:] == -1)


def test_pool_block_len_one_equals_topk():
    rng = np.random.default_rng(25)
    s = rng.integers(0, 50, 500).astype(np.float64)
    pool, n = indexer.build_pool(s, pool_blocks=37, block_len=1)
    assert n == 37 and np.array_equal(pool, indexer.topk(s, 37))


def test_pool_block_max_and_tail_block():
    s = np.zeros(21)
    s[19] = 5.0            # in the clipped tail block [16, 21)
    s[3] = 4.0
    pool, n = indexer.build_pool(s, pool_blocks=2, block_len=8)
    assert list(pool[:n]) == list(range(0, 8)) + list(range(16, 21)) and n == 13


def test_reindex_with_full_pool_equals_full_topk():
    rng = np.random.default_rng(26)
    qc = quant.e4m3_cast(rng.standard_normal((4, 64)).astype(np.float32))
    kc = quant.e4m3_cast(rng.standard_normal((3000, 64)).astype(np.float32))
    w = rng.random(4).astype(np.float32)
    S = indexer.index_scores(qc, w, kc)
    pool, n = indexer.build_pool(S, pool_blocks=400, block_len=8)    # covers all 375 blocks
    idx, _ = indexer.reindex_topk(qc, w, kc, pool, n, 256)
    assert np.array_equal(idx, indexer.topk(S, 256))


def test_planted_positions_land_in_pool():
    cfg = get_config("hier_1m", T=1 << 16, B=1, pool_blocks=512)
    L = wl.plant_layer(cfg)
    qc = quant.e4m3_cast(wl.index_query(cfg, L, 0))[-1]
    w = wl.index_weight(cfg, L, 0)[-1]
    kc = quant.e4m3_cast(wl.index_key(cfg, 0, 0, 0, cfg.T))
    S = indexer.index_scores(qc, w, kc)
    pool, n = indexer.build_pool(S, cfg.pool_blocks, cfg.pool_block_len)
    pos, _ = wl.planted(cfg, 0)
    assert np.all(np.isin(pos, pool[:n]))
