"""The fused RoPE -> attention -> inverse RoPE -> cast path (csa_attn_args
rope_cs / out_bf16) against the oracle's partial RoPE (oracle/rope.py):
every attention kernel (64 heads on tcgen05, 16 and 32 heads), one split and
many (split combine), decode and several query tokens, fp32 and bf16
output, query staged by the layer stack's prologue and converted in-kernel."""
import numpy as np
import pytest

from oracle import rope as orope
from oracle import quant as oq
from tests.parity import assert_close, assert_close_bf16
from tests.test_gpu_attn import _case

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import indexer_selected_sparse_csa2_b200 as m
    return m


def _angles(B, n_q, T, theta=160000.0):
    """RoPE tables of each query position (query t at T - n_q + t), [B, n_q, 32, 2]."""
    cs = np.zeros((B, n_q, 32, 2), np.float32)
    for b in range(B):
        for t in range(n_q):
            cs[b, t] = orope.rope_angles(T - n_q + t + 977 * b, theta)
    return cs


def _oracle_rope(kv, win, q, idx, n_win, scale, cs):
    B, n_q, H, D = q.shape
    out = np.zeros((B, n_q, H, D))
    lse = np.zeros((B, n_q, H))
    for b in range(B):
        for t in range(n_q):
            sel = idx[b, t][idx[b, t] >= 0]
            X = np.concatenate([oq.fp4_dequant_rows(kv[b][sel]), oq.fp8_window_dequant_rows(win[b][t:t + n_win])])
            out[b, t], lse[b, t] = orope.attend_rope(q[b, t], X, scale, cs[b, t])
    return out, lse


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("B,n_q,H,T,K,n_win", [
    (2, 1, 64, 5000, 2048, 128),     # decode, many splits (combine)
    (1, 1, 64, 300, 64, 16),         # decode, one split
    (1, 1, 16, 4096, 256, 128),      # 16 heads
    (2, 1, 32, 2000, 512, 128),      # 32 heads, several splits
    (1, 5, 64, 3000, 200, 32),       # several query tokens (in-kernel query conversion)
])
def test_rope_attention_matches_oracle(csa, B, n_q, H, T, K, n_win, bf16):
    kv, win, q, idx, _ = _case(5 + H + n_q, B, n_q, H, T, K, n_win)
    cs = _angles(B, n_q, T)
    scale = 1 / np.sqrt(512)
    dt = torch.bfloat16 if bf16 else torch.float32
    out = torch.full((B, n_q, H, 512), np.nan, dtype=dt, device="cuda")
    lse = torch.full((B, n_q, H), np.nan, dtype=torch.float32, device="cuda")
    a = csa.attn_args(q=torch.from_numpy(q).cuda(), kv=torch.from_numpy(kv).cuda(), idx=torch.from_numpy(idx).cuda(),
                      win=torch.from_numpy(win).cuda(), n_win=n_win, softmax_scale=scale, out=out, lse=lse,
                      rope_cs=torch.from_numpy(cs).cuda())
    csa.csa_sparse_attn(a)
    torch.cuda.synchronize()
    o, l = _oracle_rope(kv, win, q, idx, n_win, scale, cs)
    (assert_close_bf16 if bf16 else assert_close)(out.float().cpu().numpy(), o, "out")
    assert_close(lse.cpu().numpy(), l, "lse")


@pytest.mark.parametrize("bf16", [False, True])
def test_rope_in_layer_stack_staged_query(csa, bf16):
    """A decode stack: the query is staged (and rotated) by the prologue."""
    from csa_synth import get_config
    from csa_synth.device import DeviceCase
    from oracle.case import SynthCase
    from tests.parity import oracle_attend_on
    cfg = get_config("hier_1m", B=2, T=20003, pool_blocks=700, K=300)
    dc = DeviceCase(cfg)
    cs = _angles(cfg.B, 1, cfg.T)
    cs_t = torch.from_numpy(cs).cuda()
    descs = dc.layer_descs(append_rows=False)
    outs = []
    for li in range(len(cfg.layers)):
        dl = dc.layers[li]
        o = torch.full(dl.out.shape, np.nan, dtype=torch.bfloat16 if bf16 else torch.float32, device="cuda")
        descs[li].attn.out = o.data_ptr()
        descs[li].attn.out_bf16 = 1 if bf16 else 0
        descs[li].attn.rope_cs = cs_t.data_ptr()
        outs.append(o)
    csa.csa_layer_step(descs)
    torch.cuda.synchronize()
    assert csa.device_status() == 0
    for b in range(cfg.B):
        case = SynthCase(cfg, b)
        for li in range(len(cfg.layers)):
            g_idx = dc.layers[li].idx[b, 0].cpu().numpy()
            inp = case.inputs(li)
            sel = g_idx[g_idx >= 0].astype(np.int64)
            X = np.concatenate([oq.fp4_dequant_rows(case.main_entries(0, sel)),
                                oq.fp8_window_dequant_rows(inp.window[0:cfg.n_win])])
            o, l = orope.attend_rope(inp.q[0], X, cfg.softmax_scale, cs[b, 0])
            (assert_close_bf16 if bf16 else assert_close)(outs[li][b, 0].float().cpu().numpy(), o,
                                                          f"layer {li} b {b} out")
            assert_close(dc.layers[li].lse[b, 0].cpu().numpy(), l, f"layer {li} b {b} lse")
