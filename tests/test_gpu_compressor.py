"""The m-token compressor (csa_compress_kv) against the oracle (oracle/compressor.py)
and the encoded CED layer stack (2 SWA + encoder m=2 groups + decoder with
the hierarchical pool) against the oracle."""
import numpy as np
import pytest

from oracle import compressor as oc
from oracle import quant as oq
from tests.parity import check_codes_near_boundaries, topk_diff, assert_close, oracle_attend_on, check_row_format

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import indexer_selected_sparse_csa2_b200 as m
    return m


@pytest.mark.parametrize("m", [1, 2, 4])
@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("fmt", ["fp4", "e4m3"])
def test_compressor_matches_oracle(csa, m, bf16, fmt):
    rng = np.random.default_rng(7 * m + bf16 + (fmt == "fp4"))
    dim = 512 if fmt == "fp4" else 64
    n = 3001
    x = rng.standard_normal((n * m, dim)).astype(np.float32) * np.float32(1.5)
    if bf16:
        x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    g = (rng.standard_normal((n * m, dim)) * 3).astype(np.float32)
    src = torch.from_numpy(x).cuda()
    if bf16:
        src = src.to(torch.bfloat16)
    gate = torch.from_numpy(g).cuda() if m > 1 else None
    width = 288 if fmt == "fp4" else dim
    dst = torch.zeros((n, width), dtype=torch.uint8, device="cuda")
    csa.csa_compress_kv(src, gate, m, csa.CSA_FMT_FP4_E2M1_E4M3X16 if fmt == "fp4" else csa.CSA_FMT_FP8_E4M3_PLAIN,
                        dst)
    torch.cuda.synchronize()
    pooled = oc.compress(x.reshape(n, m, dim), g.reshape(n, m, dim) if m > 1 else None)
    got = dst.cpu().numpy()
    if m == 1:
        ref = oq.fp4_quant_rows(x) if fmt == "fp4" else oq.e4m3_cast(x)
        assert np.array_equal(got, ref)               # no fp32 arithmetic: bit-exact
    else:
        n_diff = check_codes_near_boundaries(got, pooled, fmt, f"m={m}")
        assert n_diff <= 1e-3 * pooled.size


def test_compressor_rejects_bad_args(csa):
    x = torch.zeros((8, 512), device="cuda")
    d = torch.zeros((4, 288), dtype=torch.uint8, device="cuda")
    with pytest.raises(csa.CsaError):
        csa.csa_compress_kv(x, None, 2, csa.CSA_FMT_FP4_E2M1_E4M3X16, d)          # m > 1 needs gates
    with pytest.raises(csa.CsaError):
        csa.csa_compress_kv(x, torch.zeros_like(x), 2, csa.CSA_FMT_FP8_E4M3_UE8M0X32, d)   # windows are not pooled


def _check_ced(csa, cfg, batches):
    from csa_synth.device import DeviceCase
    from csa_synth.configs import REINDEX, REUSE, SWA
    from oracle.case import SynthCase
    from oracle import indexer as oi
    dc = DeviceCase(cfg)
    csa.csa_layer_step(dc.layer_descs(append_rows=True))
    torch.cuda.synchronize()
    assert csa.device_status() == 0
    for b in batches:
        case = SynthCase(cfg, b)
        # the compressed caches: indexer keys and sampled main entries
        for o in cfg.owners:
            if cfg.ratio(o) == 1:
                continue
            from csa_synth import workload as wl
            E, m = cfg.entries(o), cfg.ratio(o)
            kx = wl.index_key(cfg, o, b, 0, E * m).reshape(E, m, cfg.d_I)
            kg = wl.index_gate(cfg, o, b, 0, E * m).reshape(E, m, cfg.d_I)
            check_codes_near_boundaries(dc.keys[o][b].cpu().numpy(), oc.compress(kx, kg), "e4m3", f"keys {o}")
        res = case.run(keep_scores=True)
        for li, L in enumerate(cfg.layers):
            dl = dc.layers[li]
            if L.mode == SWA:
                g_idx = np.full(cfg.K, -1, np.int32)
            else:
                src = L.reuse_from if L.mode == REUSE else li
                g_idx = dc.layers[src].idx[b, 0].cpu().numpy()
            r = res[li]
            if L.mode not in (SWA, REUSE):
                check_row_format(g_idx)
                if L.mode == REINDEX and L.pool_from >= 0:
                    P = res[L.pool_from]
                    S_full = np.full(cfg.entries(L.owner), np.nan)
                    S_full[P.pool[:P.pool_len].astype(np.int64)] = r.scores[0]
                else:
                    S_full = r.scores[0]
                topk_diff(g_idx, r.idx[0], lambda p: S_full[p])
            if np.array_equal(g_idx, r.idx[0]):
                o_out, o_lse = r.out[0], r.lse[0]
            else:
                o_out, o_lse = oracle_attend_on(case, cfg, li, 0, g_idx)
            assert_close(dl.out[b, 0].cpu().numpy(), o_out, f"layer {li} out")
            assert_close(dl.lse[b, 0].cpu().numpy(), o_lse, f"layer {li} lse")


def test_ced_stack_small(csa):
    """The 40-layer encoder-decoder stack at a small cache (8192 tokens)."""
    from csa_synth import get_config
    _check_ced(csa, get_config("ced_40", B=2, T=8192, K=512, pool_blocks=256), [0, 1])
