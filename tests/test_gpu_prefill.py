"""GPU parity of the prefill (n_q > 1, causal) indexer Top-K and of a whole
prefill layer step against the oracle."""
import numpy as np
import pytest

from oracle import indexer as oi
from oracle import quant as oq
from oracle import codecs as oc
from oracle.case import SynthCase
from csa_synth import get_config
from tests.parity import topk_diff, check_row_format, assert_close

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import indexer_selected_sparse_csa2_b200 as m
    return m


def _run(csa, kc, qc, w, K):
    B, T = kc.shape[:2]
    n_q = qc.shape[1]
    keys = torch.from_numpy(kc).cuda()
    idx = torch.full((B, n_q, K), -7, dtype=torch.int32, device="cuda")
    a = csa.index_args(keys=keys, q=torch.from_numpy(qc).cuda(), w=torch.from_numpy(w).cuda(), K=K, idx=idx,
                       n_q=n_q)
    csa.csa_index_topk(a)
    torch.cuda.synchronize()
    assert csa.device_status() == 0
    return idx.cpu().numpy()


def _check(kc, qc, w, K, got, queries=None):
    B, T = kc.shape[:2]
    n_q = qc.shape[1]
    for b in range(B):
        for t in (range(n_q) if queries is None else queries):
            n_t = T - n_q + t + 1
            S = oi.index_scores(qc[b, t], w[b, t], kc[b, :n_t])
            topk_diff(got[b, t], oi.topk(S, K), lambda p: S[p])


def _problem(seed, B, T, n_q, H_I):
    rng = np.random.default_rng(seed)
    kc = oq.e4m3_cast(rng.standard_normal((B, T, 64)).astype(np.float32))
    qc = oq.e4m3_cast(rng.standard_normal((B, n_q, H_I, 64)).astype(np.float32))
    w = rng.random((B, n_q, H_I)).astype(np.float32)
    return kc, qc, w


@pytest.mark.parametrize("B,T,n_q,H_I,K", [
    (1, 20000, 64, 8, 256),      # threshold path (visible > candidate capacity)
    (2, 9000, 45, 4, 512),       # every position fits: tau = -inf path; ragged query block
    (1, 140000, 40, 8, 2048),    # several 1024-tile key chunks
])
def test_prefill_topk(csa, B, T, n_q, H_I, K):
    kc, qc, w = _problem(T + n_q, B, T, n_q, H_I)
    got = _run(csa, kc, qc, w, K)
    qs = None if T * n_q <= 2_000_000 else [0, 1, n_q // 2, n_q - 1]
    _check(kc, qc, w, K, got, qs)


def test_prefill_fallback_when_threshold_too_high(csa):
    """High-scoring keys only inside sampled tiles (every 64th 128-row tile):
    the sampled threshold keeps fewer than K candidates, so the exact
    streaming fallback must produce the Top-K."""
    B, T, n_q, H_I, K = 1, 40000, 8, 8, 1024
    kc, qc, w = _problem(77, B, T, n_q, H_I)
    hot = oq.e4m3_cast((np.sign(oc.e4m3_decode(qc[0, 0]).sum(axis=0)) * 8.0).astype(np.float32))
    for tile in range(0, (T + 127) // 128, 64):
        kc[0, tile * 128:min(T, tile * 128 + 128)] = hot
    got = _run(csa, kc, qc, w, K)
    _check(kc, qc, w, K, got)


def test_prefill_fallback_on_overflow_with_ties(csa):
    """All keys equal: every visible position ties, the candidate buffer
    overflows, and the lowest K positions must win."""
    B, T, n_q, K = 1, 20000, 5, 300
    kc = np.full((B, T, 64), 0x38, dtype=np.uint8)
    qc = np.full((B, n_q, 8, 64), 0x38, dtype=np.uint8)
    w = np.ones((B, n_q, 8), dtype=np.float32)
    got = _run(csa, kc, qc, w, K)
    for t in range(n_q):
        assert list(got[0, t]) == list(range(K))


def test_prefill_layer_step(csa):
    """Whole prefill layer (indexer Top-K + attention over Top-K and the
    causal window) for a small chunk, checked on a few query tokens."""
    from csa_synth.device import DeviceCase
    cfg = get_config("prefill_1m", T=12000, n_q=96, K=256, W=64)
    dc = DeviceCase(cfg)
    csa.csa_layer_step(dc.layer_descs())
    torch.cuda.synchronize()
    qs = [0, 31, 32, 95]
    res = SynthCase(cfg, 0).run(queries=qs, keep_scores=True)[0]
    for r, t in enumerate(qs):
        g = dc.layers[0].idx[0, t].cpu().numpy()
        check_row_format(g)
        S = res.scores[r]
        topk_diff(g, res.idx[r], lambda p: S[p])
        if np.array_equal(g, res.idx[r]):
            assert_close(dc.layers[0].out[0, t].cpu().numpy(), res.out[r], f"query {t} out")
