"""GPU parity of sparse MLA attention vs the oracle (same indices on both sides)."""
import numpy as np
import pytest

from oracle import attention as oa
from oracle import quant as oq
from tests.parity import assert_close

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import indexer_selected_sparse_csa2_b200 as m
    return m


def _case(seed, B, n_q, H, T, K, n_win, valid=None, outliers=False, sink=False, q_gain=1.0, holes=0.0):
    rng = np.random.default_rng(seed)
    lat = rng.standard_normal((B, T, 512)).astype(np.float32)
    if outliers:
        lat[:, :, [3, 77, 300, 301, 511]] *= 20
    kv = np.stack([oq.fp4_quant_rows(lat[b]) for b in range(B)])
    rows = n_q + max(n_win, 1) - 1
    wl = rng.standard_normal((B, rows, 512)).astype(np.float32) * 2
    win = np.stack([oq.fp8_window_quant_rows(wl[b]) for b in range(B)])
    q = (rng.standard_normal((B, n_q, H, 512)) * q_gain).astype(np.float32)
    idx = np.full((B, n_q, K), -1, np.int32)
    for b in range(B):
        for t in range(n_q):
            nv = min(K, T) if valid is None else valid
            sel = np.sort(rng.choice(T, size=nv, replace=False)).astype(np.int32)
            if holes:
                sel[rng.random(nv) < holes] = -1
            idx[b, t, :nv] = sel
    sk = rng.standard_normal(H).astype(np.float32) if sink else None
    return kv, win, q, idx, sk


def _gpu(csa, kv, win, q, idx, n_win, scale, sk=None):
    B, n_q, H, D = q.shape
    out = torch.full((B, n_q, H, D), np.nan, dtype=torch.float32, device="cuda")
    lse = torch.full((B, n_q, H), np.nan, dtype=torch.float32, device="cuda")
    kv_t = torch.from_numpy(kv).cuda()
    win_t = torch.from_numpy(win).cuda()
    a = csa.attn_args(q=torch.from_numpy(q).cuda(), kv=kv_t, idx=torch.from_numpy(idx).cuda(), win=win_t,
                      n_win=n_win, softmax_scale=scale, out=out, lse=lse,
                      sink=None if sk is None else torch.from_numpy(sk).cuda())
    csa.csa_sparse_attn(a)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def _oracle(kv, win, q, idx, n_win, scale, sk=None):
    B, n_q, H, D = q.shape
    out = np.zeros((B, n_q, H, D))
    lse = np.zeros((B, n_q, H))
    for b in range(B):
        for t in range(n_q):
            sel = idx[b, t][idx[b, t] >= 0]
            X = np.concatenate([oq.fp4_dequant_rows(kv[b][sel]), oq.fp8_window_dequant_rows(win[b][t:t + n_win])])
            out[b, t], lse[b, t] = oa.attend(q[b, t], X, scale, sk)
    return out, lse


@pytest.mark.parametrize("B,n_q,H,T,K,n_win,valid", [
    (1, 1, 16, 4096, 256, 128, None),      # tiny decode shape
    (2, 1, 64, 5000, 2048, 128, None),     # full K, one token per CTA split
    (3, 1, 32, 600, 200, 7, None),         # ragged tile tail
    (1, 1, 64, 100, 256, 128, 100),        # fewer valid entries than K (-1 padding)
    (2, 3, 64, 3000, 64, 16, None),        # several query tokens, sliding window rows
    (1, 1, 64, 50, 0, 1, None),            # window only, single entry
    (1, 1, 16, 300, 1, 0, None),           # a single selected entry, no window
    (1, 40, 64, 20000, 2048, 128, None),   # prefill-like: 40 tokens, 68 tiles each
    (1, 2, 64, 3000, 1000, 100, None),     # K and window not multiples of a tile
    (1, 1, 64, 20000, 8192, 128, None),    # 130 tiles, more than 64 splits to merge
])
def test_sparse_attention(csa, B, n_q, H, T, K, n_win, valid):
    scale = float(np.float32(1 / np.sqrt(512)))
    kv, win, q, idx, _ = _case(B * 1000 + T + K, B, n_q, H, T, K, n_win, valid)
    go, gl = _gpu(csa, kv, win, q, idx, n_win, scale)
    oo, ol = _oracle(kv, win, q, idx, n_win, scale)
    assert_close(go, oo, "out")
    assert_close(gl, ol, "lse")


def test_sparse_attention_outliers_and_sink(csa):
    scale = float(np.float32(1 / np.sqrt(512)))
    kv, win, q, idx, sk = _case(9, 2, 1, 64, 8000, 2048, 128, outliers=True, sink=True)
    sk[3] = -np.inf
    go, gl = _gpu(csa, kv, win, q, idx, 128, scale, sk)
    oo, ol = _oracle(kv, win, q, idx, 128, scale, sk)
    assert_close(go, oo, "out")
    assert_close(gl, ol, "lse")


def test_no_entries_gives_zero_and_neg_inf(csa):
    kv, win, q, idx, _ = _case(11, 1, 1, 16, 10, 8, 0, valid=0)
    go, gl = _gpu(csa, kv, win, q, idx, 0, 0.1)
    assert np.all(go == 0) and np.all(np.isneginf(gl))


def test_dense_equals_full_softmax(csa):
    """K = T with no window: every cached entry is attended (dense attention)."""
    T = 640
    scale = float(np.float32(1 / np.sqrt(512)))
    kv, win, q, idx, _ = _case(12, 1, 1, 64, T, T, 0)
    assert np.array_equal(idx[0, 0], np.arange(T))
    go, gl = _gpu(csa, kv, win, q, idx, 0, scale)
    X = oq.fp4_dequant_rows(kv[0])
    oo, ol = oa.attend(q[0, 0], X, scale)
    assert_close(go[0, 0], oo, "out")
    assert_close(gl[0, 0], ol, "lse")


def test_sharp_scores_and_holes(csa):
    """Large logits (the running max moves by far more than the lazy-rescale
    threshold between tiles) and invalid (-1) entries scattered inside tiles."""
    scale = float(np.float32(1 / np.sqrt(512)))
    kv, win, q, idx, sk = _case(21, 2, 3, 64, 6000, 1536, 64, q_gain=6.0, holes=0.3, sink=True)
    go, gl = _gpu(csa, kv, win, q, idx, 64, scale, sk)
    oo, ol = _oracle(kv, win, q, idx, 64, scale, sk)
    assert_close(go, oo, "out")
    assert_close(gl, ol, "lse")


def test_mma_sync_kernel_for_64_heads(csa):
    """The mma.sync kernel that 64 heads run on when CSA_ATTN_MMA_SYNC=1 (the
    tcgen05 kernel is the default) passes the same cases."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, CSA_ATTN_MMA_SYNC="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", __file__, "-k", "not mma_sync_kernel"],
                       env=env, capture_output=True, text=True, cwd=os.path.dirname(os.path.dirname(__file__)))
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
