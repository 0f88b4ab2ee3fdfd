"""Context-parallel decode kernels on one GPU, the ranks simulated by shards
of one device case (the exchange is a stack in rank order, as an all-gather
returns it), against the oracle (oracle/context_parallel.py and the
single-rank oracle)."""
import numpy as np
import pytest

from csa_synth import get_config
from oracle import context_parallel as cpr
from oracle import indexer as oi
from oracle.case import SynthCase
from tests.parity import topk_diff, assert_close, oracle_attend_on

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import indexer_selected_sparse_csa2_b200 as m
    return m


@pytest.mark.parametrize("R,B,Kl,K", [(1, 1, 64, 64), (3, 2, 300, 256), (8, 3, 512, 1000), (5, 1, 40, 256)])
def test_merge_equals_oracle_merge(csa, R, B, Kl, K):
    """Given the same (score, position) pairs the merge is bit-exact (heavy
    ties across ranks; ranks whose lists are partly padding)."""
    rng = np.random.default_rng(R * 100 + K)
    T = R * 4 * Kl
    bounds = cpr.shard_bounds(T, R)
    ps = np.full((R, B, Kl), -np.inf, np.float32)
    pp = np.full((R, B, Kl), -1, np.int32)
    parts_b = [[] for _ in range(B)]
    for r, (t0, t1) in enumerate(bounds):
        for b in range(B):
            S = rng.integers(0, 30, t1 - t0).astype(np.float32) * np.float32(0.25)
            if r == 1:
                S = S[: max(1, Kl // 3)]          # a short shard: its list is partly padding
            s, p = cpr.local_topk(S.astype(np.float64), t0, Kl)
            order = np.argsort(p)                  # the local lists are ascending by position
            ps[r, b, :s.size] = s[order]
            pp[r, b, :p.size] = p[order]
            parts_b[b].append((s, p))
    idx = torch.full((B, K), -7, dtype=torch.int32, device="cuda")
    csa.csa_cp_merge_topk(torch.from_numpy(ps).cuda(), torch.from_numpy(pp).cuda(), K, idx)
    torch.cuda.synchronize()
    got = idx.cpu().numpy()
    for b in range(B):
        assert np.array_equal(got[b], cpr.merge_topk(parts_b[b], K)), b


@pytest.mark.parametrize("sink", [False, True])
def test_combine_equals_oracle_combine(csa, sink):
    rng = np.random.default_rng(11 + sink)
    R, B, H = 5, 2, 64
    outs = rng.standard_normal((R, B, H, 512)).astype(np.float32) * 3
    lses = rng.standard_normal((R, B, H)).astype(np.float32) * 4
    lses[2, 0, :] = -np.inf                      # a rank with no entries
    sk = rng.standard_normal(H).astype(np.float32) if sink else None
    out = torch.empty((B, H, 512), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    csa.csa_cp_combine(torch.from_numpy(outs).cuda(), torch.from_numpy(lses).cuda(), out, lse,
                       sink=torch.from_numpy(sk).cuda() if sink else None)
    torch.cuda.synchronize()
    for b in range(B):
        o, l = cpr.combine([(outs[r, b].astype(np.float64), lses[r, b].astype(np.float64)) for r in range(R)], sk)
        assert_close(out[b].cpu().numpy(), o, f"b {b} out")
        assert_close(lse[b].cpu().numpy(), l, f"b {b} lse")


def test_localize(csa):
    idx = torch.tensor([[5, 17, 99, 100, 250, -1]], dtype=torch.int32, device="cuda")
    loc = torch.empty_like(idx)
    csa.csa_cp_localize(idx, 17, 100, loc)
    torch.cuda.synchronize()
    assert loc.cpu().tolist() == [[-1, 0, 82, -1, -1, -1]]


@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_sharded_decode_matches_single_rank_oracle(csa, world):
    """A whole sharded decode step, ranks run one after another on this GPU:
    the global Top-K by the score-tie rule against the single-rank oracle,
    and the combined attention against the oracle's attention over the
    selected set."""
    from csa_synth.device import DeviceCase
    from indexer_selected_sparse_csa2_b200.context_parallel import DeviceShard, shard_bounds
    cfg = get_config("decode_64k", B=2, T=20000)
    dc = DeviceCase(cfg)
    L = dc.layers[0]
    shards = []
    for t0, t1 in shard_bounds(cfg.T, world):
        shards.append((t0, t1, DeviceShard(dc.keys[0][:, t0:t1], dc.kv[0][:, t0:t1], L.q, L.qI, L.w, L.win,
                                           cfg.n_win, cfg.K, cfg.softmax_scale)))
    pairs = [sh.local_topk(t0, t1) for t0, t1, sh in shards]
    gs = torch.stack([p[0] for p in pairs])
    gp = torch.stack([p[1] for p in pairs])
    idx = shards[0][2].merge(gs, gp)
    parts = [sh.attend(idx, t0, t1, r == world - 1) for r, (t0, t1, sh) in enumerate(shards)]
    out, lse = shards[0][2].combine(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    torch.cuda.synchronize()
    assert csa.device_status() == 0
    for b in range(cfg.B):
        case = SynthCase(cfg, b)
        res = case.run(keep_scores=True)[0]
        g_idx = idx[b].cpu().numpy()
        topk_diff(g_idx, res.idx[0], lambda p: res.scores[0][p])
        if np.array_equal(g_idx, res.idx[0]):
            o_out, o_lse = res.out[0], res.lse[0]
        else:
            o_out, o_lse = oracle_attend_on(case, cfg, 0, 0, g_idx)
        assert_close(out[b].cpu().numpy(), o_out, f"world {world} b {b} out")
        assert_close(lse[b].cpu().numpy(), o_lse, f"world {world} b {b} lse")
