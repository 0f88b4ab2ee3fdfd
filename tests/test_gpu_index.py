"""GPU parity of indexer scoring, Top-K and the candidate pool vs the oracle."""
import numpy as np
import pytest

from oracle import indexer as oi
from oracle import quant as oq
from tests.parity import topk_diff, check_row_format

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import indexer_selected_sparse_csa2_b200 as m
    return m


def _problem(seed, B, T, H_I, key_scale=1.0):
    rng = np.random.default_rng(seed)
    kf = (rng.standard_normal((B, T, 64)) * key_scale).astype(np.float32)
    qf = rng.standard_normal((B, 1, H_I, 64)).astype(np.float32)
    w = rng.random((B, 1, H_I)).astype(np.float32)
    return oq.e4m3_cast(kf), oq.e4m3_cast(qf), w


def _run_index(csa, kc, qc, w, K, pool_out=False, pool_blocks=2048, pool_block_len=8, pool=None,
               pool_len=None, scores=True):
    B, T = kc.shape[:2]
    keys = torch.from_numpy(kc).cuda()
    q = torch.from_numpy(qc).cuda()
    wt = torch.from_numpy(w).cuda()
    idx = torch.full((B, 1, K), -7, dtype=torch.int32, device="cuda")
    n = pool.shape[1] if pool is not None else T
    sc = torch.zeros((B, n), dtype=torch.float32, device="cuda") if scores else None
    po = pl = None
    if pool_out:
        po = torch.full((B, pool_blocks * pool_block_len), -7, dtype=torch.int32, device="cuda")
        pl = torch.zeros(B, dtype=torch.int32, device="cuda")
    pin = plen = None
    if pool is not None:
        pin = torch.from_numpy(pool).cuda()
        plen = torch.from_numpy(pool_len).cuda()
    a = csa.index_args(keys=keys, q=q, w=wt, K=K, idx=idx, pool_out=po, pool_out_len=pl,
                       pool_blocks=pool_blocks, pool_block_len=pool_block_len, pool=pin, pool_len=plen,
                       scores=sc)
    csa.csa_index_topk(a)
    torch.cuda.synchronize()
    res = {"idx": idx.cpu().numpy()[:, 0]}
    if sc is not None:
        res["scores"] = sc.cpu().numpy()
    if pool_out:
        res["pool"] = po.cpu().numpy()
        res["pool_len"] = pl.cpu().numpy()
    return res


@pytest.mark.parametrize("B,T,H_I,K", [(1, 4096, 4, 256), (3, 300, 8, 64), (2, 1, 8, 16),
                                       (1, 17, 1, 64), (2, 5000, 5, 4096), (1, 70000, 8, 2048)])
def test_decode_scores_and_topk(csa, B, T, H_I, K):
    kc, qc, w = _problem(100 + T, B, T, H_I)
    res = _run_index(csa, kc, qc, w, K)
    for b in range(B):
        S = oi.index_scores(qc[b, 0], w[b, 0], kc[b])
        # scores: fp32 of an exact value, within fp32 summation error
        err = np.abs(res["scores"][b].astype(np.float64) - S)
        assert np.all(err <= 1e-5 * np.maximum(np.abs(S), 1e-3)), err.max()
        ora = oi.topk(S, K)
        topk_diff(res["idx"][b], ora, lambda p: S[p])


def test_topk_with_massive_ties(csa):
    """All keys equal: every score ties, so the K lowest positions win."""
    B, T, K = 2, 20000, 300
    kc = np.full((B, T, 64), 0x38, dtype=np.uint8)
    qc = np.full((B, 1, 8, 64), 0x38, dtype=np.uint8)
    w = np.ones((B, 1, 8), dtype=np.float32)
    res = _run_index(csa, kc, qc, w, K)
    for b in range(B):
        assert list(res["idx"][b]) == list(range(K))


def test_zero_scores_ties(csa):
    """Negative dot products give score 0 under ReLU: ties at zero pick lowest positions."""
    B, T, K = 1, 3000, 1000
    rng = np.random.default_rng(7)
    kc = oq.e4m3_cast(-np.abs(rng.standard_normal((B, T, 64))).astype(np.float32))
    kc[0, 100:400] = oq.e4m3_cast(np.abs(rng.standard_normal((300, 64))).astype(np.float32))
    qc = oq.e4m3_cast(np.abs(rng.standard_normal((B, 1, 4, 64))).astype(np.float32))
    w = rng.random((B, 1, 4)).astype(np.float32)
    res = _run_index(csa, kc, qc, w, K)
    S = oi.index_scores(qc[0, 0], w[0, 0], kc[0])
    ora = oi.topk(S, K)
    assert np.array_equal(res["idx"][0], ora)


@pytest.mark.parametrize("T,bl,nblk", [(20000, 8, 256), (1000, 8, 2048), (4099, 4, 300),
                                       (5000, 16, 100), (777, 1, 50), (3333, 2, 900)])
def test_pool_build(csa, T, bl, nblk):
    B = 2
    kc, qc, w = _problem(200 + T, B, T, 8)
    res = _run_index(csa, kc, qc, w, 64, pool_out=True, pool_blocks=nblk, pool_block_len=bl)
    for b in range(B):
        S = oi.index_scores(qc[b, 0], w[b, 0], kc[b])
        pool, n = oi.build_pool(S, nblk, bl)
        gp, gn = res["pool"][b], int(res["pool_len"][b])
        check_row_format(gp)
        assert gn == int((gp >= 0).sum())
        bm = oi.block_max(S, bl)
        gblk = np.unique(gp[:gn] // bl)
        oblk = np.unique(pool[:n] // bl)
        topk_diff(np.concatenate([gblk, -np.ones(nblk - gblk.size, np.int64)]),
                  np.concatenate([oblk, -np.ones(nblk - oblk.size, np.int64)]), lambda p: bm[p])
        if np.array_equal(gblk, oblk):
            assert gn == n and np.array_equal(gp, pool)


def test_reindex_over_pool(csa):
    B, T, K = 2, 30000, 512
    kc, qc, w = _problem(300, B, T, 8)
    rng = np.random.default_rng(301)
    cap = 8 * 700
    pools, lens = [], []
    for b in range(B):
        blocks = np.sort(rng.choice(T // 8, size=700 - 3 * b, replace=False))
        pos = (blocks[:, None] * 8 + np.arange(8)).reshape(-1).astype(np.int32)
        p = np.full(cap, -1, np.int32)
        p[:pos.size] = pos
        pools.append(p)
        lens.append(pos.size)
    pool = np.stack(pools)
    pool_len = np.array(lens, np.int32)
    res = _run_index(csa, kc, qc, w, K, pool=pool, pool_len=pool_len)
    for b in range(B):
        ora, S = oi.reindex_topk(qc[b, 0], w[b, 0], kc[b], pool[b], int(pool_len[b]), K)
        full = oi.index_scores(qc[b, 0], w[b, 0], kc[b])
        topk_diff(res["idx"][b], ora, lambda p: full[p])
        n = int(pool_len[b])
        err = np.abs(res["scores"][b, :n] - S)
        assert np.all(err <= 1e-5 * np.maximum(np.abs(S), 1e-3))


@pytest.mark.parametrize("n_blocks,lens", [(9000, (72000, 71111)), (700, (0, 5600))])
def test_reindex_pool_sizes(csa, n_blocks, lens):
    """Pools longer than the fused pool kernel takes (gathered scoring, then the
    select over the scores) and a row whose pool is empty (all -1)."""
    B, T, K = 2, 200000, 512
    kc, qc, w = _problem(400 + n_blocks, B, T, 8)
    rng = np.random.default_rng(401)
    cap = 8 * n_blocks
    pools = []
    for b in range(B):
        blocks = np.sort(rng.choice(T // 8, size=(lens[b] + 7) // 8, replace=False))
        pos = (blocks[:, None] * 8 + np.arange(8)).reshape(-1)[:lens[b]].astype(np.int32)
        p = np.full(cap, -1, np.int32)
        p[:pos.size] = pos
        pools.append(p)
    pool = np.stack(pools)
    pool_len = np.array(lens, np.int32)
    res = _run_index(csa, kc, qc, w, K, pool=pool, pool_len=pool_len)
    for b in range(B):
        n = int(pool_len[b])
        if n == 0:
            assert np.all(res["idx"][b] == -1)
            continue
        ora, S = oi.reindex_topk(qc[b, 0], w[b, 0], kc[b], pool[b], n, K)
        full = oi.index_scores(qc[b, 0], w[b, 0], kc[b])
        topk_diff(res["idx"][b], ora, lambda p: full[p])


def _run_topk(csa, s, K):
    st = torch.from_numpy(s).cuda()
    idx = torch.full((s.shape[0], K), -7, dtype=torch.int32, device="cuda")
    csa.csa_topk_scores(st, K, idx)
    torch.cuda.synchronize()
    return idx.cpu().numpy()


@pytest.mark.parametrize("B,n,K", [(1, 1, 1), (2, 300, 64), (3, 257, 400), (2, 100000, 2048),
                                   (1, 1 << 20, 2048), (4, 50000, 1)])
def test_topk_scores_bit_exact(csa, B, n, K):
    rng = np.random.default_rng(n + K)
    s = rng.integers(-20, 20, size=(B, n)).astype(np.float32) * np.float32(0.5)   # heavy ties
    s[:, ::7] = rng.standard_normal((B, s[:, ::7].shape[1])).astype(np.float32)
    s[0, :3] = np.float32([-0.0, 0.0, -0.0])[:min(3, n)]
    got = _run_topk(csa, s, K)
    for b in range(B):
        assert np.array_equal(got[b], oi.topk(s[b].astype(np.float64), K)), b


def test_topk_scores_candidate_overflow_path(csa):
    """More threshold-bin candidates than fit in shared memory (global list path)."""
    B, n, K = 1, 400000, 5000
    s = np.zeros((B, n), np.float32)
    s[0, 1000:1100] = 1.0
    got = _run_topk(csa, s, K)
    assert np.array_equal(got[0], oi.topk(s[0].astype(np.float64), K))


def test_zz_no_device_wait_timeouts(csa):
    """No bounded device wait of the kernels above ran out (status 0)."""
    torch.cuda.synchronize()
    assert csa.device_status() == 0
