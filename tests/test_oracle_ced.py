"""Pins for the oracle's encoder-decoder stack features (CPU only): window-only
(SWA) layers, owners whose caches hold one entry per m tokens, and the
40-layer pattern."""
import numpy as np

from csa_synth import get_config
from csa_synth import workload as wl
from csa_synth.configs import LayerSpec, FULL, REUSE, SWA, REINDEX
from oracle import quant as oq
from oracle import indexer as oi
from oracle import compressor as oc
from oracle.attention import attend
from oracle.case import SynthCase
from oracle.layers import LayerInputs, run_stack


def _inputs(rng, H=4, H_I=2, n_win=16):
    return LayerInputs(qI=oq.e4m3_cast(rng.standard_normal((1, H_I, 64)).astype(np.float32)),
                       w=rng.random((1, H_I)).astype(np.float32),
                       q=rng.standard_normal((1, H, 512)).astype(np.float32),
                       window=oq.fp8_window_quant_rows(rng.standard_normal((n_win, 512)).astype(np.float32)))


def test_swa_layer_attends_to_its_window_only():
    rng = np.random.default_rng(1)
    inp = _inputs(rng)
    res = run_stack([LayerSpec(SWA, 0)], 100, 1, 8, 16, 0.05, keys=None, main_entries=None,
                    inputs=lambda li: inp)[0]
    o, l = attend(inp.q[0], oq.fp8_window_dequant_rows(inp.window), 0.05)
    assert np.all(res.idx == -1)
    assert np.allclose(res.out[0], o, rtol=1e-14, atol=1e-14) and np.allclose(res.lse[0], l, rtol=1e-14)


def test_compressed_owner_selects_among_its_entries():
    rng = np.random.default_rng(2)
    T, K = 400, 30
    E = T // 2
    keys = oq.e4m3_cast(rng.standard_normal((E, 64)).astype(np.float32))
    lat = rng.standard_normal((E, 512)).astype(np.float32)
    inp = _inputs(rng)
    res = run_stack([LayerSpec(FULL, 0, m=2)], T, 1, K, 16, 0.05, keys=lambda o: keys,
                    main_entries=lambda o, p: oq.fp4_quant_rows(lat[p]), inputs=lambda li: inp,
                    owner_len=lambda o: E, keep_scores=True)[0]
    S = oi.index_scores(inp.qI[0], inp.w[0], keys)
    assert np.array_equal(res.idx[0], oi.topk(S, K))
    assert res.idx[0].max() < E and res.scores[0].shape == (E,)


def test_case_pools_consecutive_token_pairs():
    cfg = get_config("ced_40", B=1, T=64, K=8, pool_blocks=4)
    case = SynthCase(cfg, 0)
    o = 8                                             # an encoder owner (m = 2)
    x = wl.main_latent(cfg, o, 0, 0, cfg.T)
    g = wl.main_gate(cfg, o, 0, 0, cfg.T)
    for j in (0, 5, cfg.entries(o) - 1):
        ref = oq.fp4_quant_rows(oc.compress(x[2 * j:2 * j + 2][None], g[2 * j:2 * j + 2][None]).astype(np.float32))
        assert np.array_equal(case.main_entries(o, np.array([j])), ref)
    kx = wl.index_key(cfg, o, 0, 0, cfg.T)
    kg = wl.index_gate(cfg, o, 0, 0, cfg.T)
    ref = oq.e4m3_cast(oc.compress(kx.reshape(-1, 2, 64), kg.reshape(-1, 2, 64)).astype(np.float32))
    assert np.array_equal(case.keys(o), ref)


def test_ced_40_pattern():
    cfg = get_config("ced_40")
    modes = [L.mode for L in cfg.layers]
    assert len(modes) == 40 and modes[:2] == [SWA, SWA]
    assert [i for i, L in enumerate(cfg.layers) if L.mode == FULL] == [2, 8, 14, 20]
    assert [i for i, L in enumerate(cfg.layers) if L.mode == REINDEX] == [24, 28, 32, 36]
    assert sum(m == REUSE for m in modes) == 15 + 3 + 12
    assert [cfg.ratio(o) for o in cfg.owners] == [2, 2, 2, 1] and cfg.owners == [2, 8, 14, 20]
    # every Reuse layer reads its group's indices and its group's owner's caches
    for i, L in enumerate(cfg.layers):
        if L.mode == REUSE:
            src = cfg.layers[L.reuse_from]
            assert src.mode in (FULL, REINDEX) and src.owner == L.owner
