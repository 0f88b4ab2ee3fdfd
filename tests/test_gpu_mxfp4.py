"""MXFP4 indexer keys on the GPU (the pages' production indexer: E2M1 with one
E8M0 scale per 32 channels, 32 heads x 128, top-512) against the oracle
(oracle/mxfp4.py): the encoder bit-exact, the tcgen05 scorer's scores within
fp32 accumulation error of the exact ones, the Top-K by the score-tie rule,
and the decode_mx workload end to end."""
import os

import numpy as np
import pytest

from oracle import mxfp4 as omx
from oracle import quant as oq
from tests.parity import topk_diff, assert_close, check_row_format, oracle_attend_on

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import indexer_selected_sparse_csa2_b200 as m
    return m


def _encode(csa, x, bf16=False):
    src = torch.from_numpy(x).cuda()
    if bf16:
        src = src.to(torch.bfloat16)
    n, dim = x.shape
    codes = torch.zeros((n, dim // 2), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((n, dim // 32), dtype=torch.uint8, device="cuda")
    csa.csa_quant_mxfp4(src, codes, scales)
    torch.cuda.synchronize()
    return np.concatenate([codes.cpu().numpy(), scales.cpu().numpy()], axis=1)


@pytest.mark.parametrize("bf16", [False, True])
def test_encoder_bit_exact(csa, bf16):
    rng = np.random.default_rng(3 + bf16)
    x = (rng.standard_normal((5000, 128)) * np.exp(rng.uniform(-12, 12, (5000, 1)))).astype(np.float32)
    x[0] = 0.0
    x[1, :32] = 6.0
    x[2, :32] = 1e-30
    ties = rng.choice([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], size=128).astype(np.float32)
    x[3] = ties * np.float32(2.0 ** rng.integers(-3, 4))
    if bf16:
        x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(_encode(csa, x, bf16), omx.mxfp4_quant_rows(x))


def test_encoder_worked_examples(csa):
    """The hand-computed blocks of tests/golden/mxfp4_block_examples.txt."""
    rows = {"all_ones": [1.0] * 32, "all_zero": [0.0] * 32, "six_block": [6, 3, -1.5, 0.25] + [0] * 28,
            "over_six": [6.5, 5, -0.75] + [0] * 29, "small": [0.1, -0.05] + [0] * 30}
    x = np.zeros((len(rows), 128), np.float32)
    names = list(rows)
    for i, n in enumerate(names):
        x[i, :32] = np.float32(rows[n])
    got = _encode(csa, x)
    for ln in open(os.path.join(GOLDEN, "mxfp4_block_examples.txt")):
        if ln.startswith("#") or not ln.strip():
            continue
        name, sb, codes, _ = ln.split()
        g = got[names.index(name)]
        assert g[64] == int(sb, 16), name
        first4 = "".join(f"{(g[i // 2] >> (4 * (i % 2))) & 0xF:X}" for i in range(4))
        assert first4 == codes.upper(), (name, first4, codes)


def _index(csa, entries, qc, w, K, scales_layout=True):
    B, T = entries.shape[:2]
    codes = torch.from_numpy(np.ascontiguousarray(entries[:, :, :64])).cuda()
    scales = torch.from_numpy(np.ascontiguousarray(entries[:, :, 64:])).cuda()
    q = torch.from_numpy(qc).cuda()
    wt = torch.from_numpy(w).cuda()
    idx = torch.full((B, 1, K), -7, dtype=torch.int32, device="cuda")
    sc = torch.zeros((B, T), dtype=torch.float32, device="cuda")
    csa.csa_index_topk(csa.index_args(keys=codes, key_scales=scales, q=q, w=wt, K=K, idx=idx, scores=sc))
    torch.cuda.synchronize()
    return idx.cpu().numpy()[:, 0], sc.cpu().numpy()


@pytest.mark.parametrize("B,T,K", [(1, 700, 64), (3, 5000, 512), (2, 129, 512), (1, 40000, 512)])
def test_scores_and_topk(csa, B, T, K):
    rng = np.random.default_rng(T + K)
    entries = np.stack([omx.mxfp4_quant_rows((rng.standard_normal((T, 128)) *
                                              np.exp(rng.uniform(-2, 2, (T, 4))).repeat(32, 1)).astype(np.float32))
                        for _ in range(B)])
    qc = oq.e4m3_cast(rng.standard_normal((B, 1, 32, 128)).astype(np.float32))
    w = rng.random((B, 1, 32)).astype(np.float32)
    idx, sc = _index(csa, entries, qc, w, K)
    for b in range(B):
        S = omx.mx_index_scores(qc[b, 0], w[b, 0], entries[b])
        err = np.abs(sc[b].astype(np.float64) - S)
        assert np.all(err <= 1e-5 * np.maximum(np.abs(S), 1e-3)), err.max()
        check_row_format(idx[b])
        from oracle import indexer as oi
        topk_diff(idx[b], oi.topk(S, K), lambda p: S[p])


def test_decode_mx_workload(csa):
    """The decode_mx workload (8 sequences x 65,536 positions) through the
    layer step, checked on two sequences."""
    from csa_synth import get_config
    from csa_synth.device import DeviceCase
    from oracle.case import SynthCase
    cfg = get_config("decode_mx")
    dc = DeviceCase(cfg)
    csa.csa_layer_step(dc.layer_descs(append_rows=True))
    torch.cuda.synchronize()
    assert csa.device_status() == 0
    for b in (0, cfg.B - 1):
        case = SynthCase(cfg, b, threads=os.cpu_count() or 4, dense_latents=True)
        rows = np.array([0, 1, cfg.T // 2, cfg.T - 1])
        got = np.concatenate([dc.keys[0][b].cpu().numpy()[rows], dc.key_scales[0][b].cpu().numpy()[rows]], axis=1)
        assert np.array_equal(got, case.keys(0)[rows])
        res = case.run(keep_scores=True)[0]
        g_idx = dc.layers[0].idx[b, 0].cpu().numpy()
        topk_diff(g_idx, res.idx[0], lambda p: res.scores[0][p])
        if np.array_equal(g_idx, res.idx[0]):
            o_out, o_lse = res.out[0], res.lse[0]
        else:
            o_out, o_lse = oracle_attend_on(case, cfg, 0, 0, g_idx)
        assert_close(dc.layers[0].out[b, 0].cpu().numpy(), o_out, f"b {b} out")
        assert_close(dc.layers[0].lse[b, 0].cpu().numpy(), o_lse, f"b {b} lse")


def test_mx_index_rejects_unsupported(csa):
    codes = torch.zeros((1, 100, 64), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((1, 100, 4), dtype=torch.uint8, device="cuda")
    q = torch.zeros((1, 1, 8, 128), dtype=torch.uint8, device="cuda")     # 8 heads: not the MXFP4 indexer shape
    w = torch.zeros((1, 1, 8), dtype=torch.float32, device="cuda")
    idx = torch.zeros((1, 1, 16), dtype=torch.int32, device="cuda")
    with pytest.raises(csa.CsaError):
        csa.csa_index_topk(csa.index_args(keys=codes, key_scales=scales, q=q, w=w, K=16, idx=idx))
