"""csa_index_topk_noalloc: the indexer + Top-K call for callers that cannot
allocate device memory (its scratch is a fixed array inside the library).

Checked through the C ABI against csa_index_topk with a caller workspace, on
two calls in a row (the array keeps the previous call's contents, so the
second call shows that everything that must start cleared is cleared).  This
file is collected last so a stop-at-first-failure run has already run every
other test; it also passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import indexer_selected_sparse_csa2_b200 as m
    return m


def _problem(seed, B, T, H_I):
    from oracle import quant as oq
    rng = np.random.default_rng(seed)
    kc = oq.e4m3_cast(rng.standard_normal((B, T, 64)).astype(np.float32))
    qc = oq.e4m3_cast(rng.standard_normal((B, 1, H_I, 64)).astype(np.float32))
    w = rng.random((B, 1, H_I)).astype(np.float32)
    return (torch.from_numpy(kc).cuda(), torch.from_numpy(qc).cuda(), torch.from_numpy(w).cuda())


def _args(csa, keys, q, w, K, pool_out=False):
    B = keys.shape[0]
    idx = torch.full((B, 1, K), -7, dtype=torch.int32, device="cuda")
    sc = torch.zeros((B, keys.shape[1]), dtype=torch.float32, device="cuda")
    po = pl = None
    if pool_out:
        po = torch.full((B, 64 * 8), -7, dtype=torch.int32, device="cuda")
        pl = torch.zeros(B, dtype=torch.int32, device="cuda")
    a = csa.index_args(keys=keys, q=q, w=w, K=K, idx=idx, scores=sc, pool_out=po, pool_out_len=pl,
                       pool_blocks=64, pool_block_len=8)
    return a, idx, sc, po, pl


@pytest.mark.parametrize("B,T,H_I,K,pool", [(2, 20000, 8, 512, True), (3, 4099, 4, 256, False)])
def test_noalloc_matches_workspace_call_twice(csa, B, T, H_I, K, pool):
    stream = torch.cuda.current_stream()
    for call, seed in enumerate((1, 2)):               # two calls in a row, different inputs
        keys, q, w = _problem(100 * call + seed, B, T, H_I)
        a_ref, idx_ref, sc_ref, po_ref, pl_ref = _args(csa, keys, q, w, K, pool)
        need = csa.csa_index_workspace_size(a_ref)
        assert 0 < need <= csa.csa_index_noalloc_capacity()
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        st = csa._index(ctypes.byref(a_ref), ws.data_ptr(), need, stream.cuda_stream)
        assert st == csa.CSA_OK
        a_na, idx_na, sc_na, po_na, pl_na = _args(csa, keys, q, w, K, pool)
        st = csa._index_noalloc(ctypes.byref(a_na), stream.cuda_stream)   # through the C ABI
        assert st == csa.CSA_OK, csa.status_string(st)
        torch.cuda.synchronize()
        # same kernels on the same inputs: identical scores and index sets
        assert torch.equal(idx_na, idx_ref)
        assert torch.equal(sc_na, sc_ref)
        if pool:
            assert torch.equal(po_na, po_ref) and torch.equal(pl_na, pl_ref)
        assert int((idx_na >= 0).sum()) == B * min(K, T)


def test_noalloc_rejects_oversized_request(csa):
    keys = torch.zeros((8, 1 << 19, 64), dtype=torch.uint8, device="cuda")   # needs > 16 MiB scratch
    q = torch.zeros((8, 1, 8, 64), dtype=torch.uint8, device="cuda")
    w = torch.zeros((8, 1, 8), dtype=torch.float32, device="cuda")
    a, *_ = _args(csa, keys, q, w, 16)
    assert csa.csa_index_workspace_size(a) > csa.csa_index_noalloc_capacity()
    assert csa._index_noalloc(ctypes.byref(a), torch.cuda.current_stream().cuda_stream) == csa.CSA_ERR_WORKSPACE
