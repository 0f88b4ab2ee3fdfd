"""Pins for the oracle's sparse attention, layer modes and byte accounting (CPU only)."""
import os

import numpy as np
import torch

from oracle import attention, quant, indexer, accounting
from oracle.case import SynthCase
from oracle.layers import LayerInputs, run_stack
from csa_synth import get_config
from csa_synth.configs import LayerSpec, FULL, REINDEX, REUSE

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def check_dense(attend_fn):
    rng = np.random.default_rng(31)
    T, H, D = 97, 8, 512
    cache = quant.fp4_dequant_rows(quant.fp4_quant_rows(rng.standard_normal((T, D)).astype(np.float32)))
    q = rng.standard_normal((H, D)).astype(np.float32)
    scale = 1 / np.sqrt(D)
    out, lse = attend_fn(q, cache, scale)
    qt = torch.from_numpy(q.astype(np.float64))[None, :, None, :]
    kv = torch.from_numpy(cache)[None, None].expand(1, H, T, D)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kv, kv, scale=float(np.float32(scale)))
    ref = ref[0, :, 0].numpy()
    ref_lse = torch.logsumexp(torch.from_numpy(q.astype(np.float64)) @ torch.from_numpy(cache).T
                              * float(np.float32(scale)), dim=1).numpy()
    return np.allclose(out, ref, rtol=1e-12, atol=1e-12) and np.allclose(lse, ref_lse, rtol=1e-12)


def test_attention_equals_dense_sdpa():
    assert check_dense(attention.attend)


def test_attention_mutation_missing_scale_is_caught():
    assert not check_dense(lambda q, X, s, sink=None: attention.attend(q, X, 1.0, sink))


def test_attention_single_entry_returns_it():
    rng = np.random.default_rng(32)
    x = quant.fp4_dequant_rows(quant.fp4_quant_rows(rng.standard_normal((1, 512)).astype(np.float32)))
    out, _ = attention.attend(rng.standard_normal((4, 512)).astype(np.float32), x, 0.04)
    assert np.array_equal(out, np.repeat(x, 4, axis=0))


def test_attention_sink_is_extra_denominator_term():
    rng = np.random.default_rng(33)
    X = rng.standard_normal((20, 512))
    q = rng.standard_normal((3, 512)).astype(np.float32)
    sink = np.float32([0.5, -np.inf, 3.0])
    out, lse = attention.attend(q, X, 0.05, sink)
    logits = torch.from_numpy(q.astype(np.float64)) @ torch.from_numpy(X).T * float(np.float32(0.05))
    full = torch.cat([logits, torch.from_numpy(sink.astype(np.float64))[:, None]], dim=1)
    p = torch.softmax(full, dim=1)[:, :20]
    assert np.allclose(out, (p @ torch.from_numpy(X)).numpy(), rtol=1e-12, atol=1e-13)
    assert np.allclose(lse, torch.logsumexp(full, dim=1).numpy(), rtol=1e-12)


def test_attention_no_entries():
    out, lse = attention.attend(np.ones((2, 512), np.float32), np.zeros((0, 512)), 0.1)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def _small(name, **kw):
    base = dict(T=700, K=64, W=16, H=16, B=1)
    base.update(kw)
    return get_config(name, **base)


def test_reuse_equals_recompute_with_same_indices():
    cfg = _small("stack_128k")
    res = SynthCase(cfg, 0).run()
    # layer 2 reuses layer 1's indices; recompute attention with those indices directly
    case = SynthCase(cfg, 0)
    inp = case.inputs(2)
    sel = res[1].idx[0]
    sel = sel[sel >= 0]
    Xm = quant.fp4_dequant_rows(case.main_entries(0, sel))
    Xw = quant.fp8_window_dequant_rows(inp.window[0:cfg.n_win])
    out, lse = attention.attend(inp.q[0], np.concatenate([Xm, Xw]), cfg.softmax_scale)
    assert np.array_equal(res[2].idx, res[1].idx)
    assert np.array_equal(res[2].out[0], out) and np.array_equal(res[2].lse[0], lse)


def test_reindex_with_full_queries_gives_full_indices():
    cfg = _small("stack_128k", layers=[LayerSpec(FULL, 0), LayerSpec(REINDEX, 0)])
    case = SynthCase(cfg, 0)
    same = case.inputs(0)
    res = run_stack(cfg.layers, cfg.T, cfg.n_q, cfg.K, cfg.n_win, cfg.softmax_scale,
                    case.keys, case.main_entries, lambda li: same)
    assert np.array_equal(res[0].idx, res[1].idx)
    assert np.array_equal(res[0].out, res[1].out)


def test_prefill_query_equals_decode_with_truncated_cache():
    cfg = _small("prefill_1m", T=900, n_q=40, K=32)
    case = SynthCase(cfg, 0)
    res = case.run(queries=[0, 17, 39])
    for r, t in enumerate([0, 17, 39]):
        n_t = cfg.T - cfg.n_q + t + 1
        S = indexer.index_scores(case.inputs(0).qI[t], case.inputs(0).w[t], case.keys(0)[:n_t])
        assert np.array_equal(res[0].idx[r], indexer.topk(S, cfg.K))
        assert res[0].idx[r].max() <= n_t - 1


def test_k_at_least_context_selects_everything():
    cfg = _small("tiny_decode", T=50, K=64)
    res = SynthCase(cfg, 0).run()
    assert list(res[0].idx[0]) == list(range(50)) + [-1] * 14


def test_byte_accounting_matches_pages():
    want = {}
    with open(os.path.join(GOLDEN, "byte_accounting.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, v = line.split()
                want[k] = int(v)
    assert accounting.MAIN_KV_BYTES == want["main_kv_entry_bytes"] == quant.FP4_ENTRY_BYTES
    assert accounting.INDEXER_K_BYTES == want["indexer_k_entry_bytes"]
    assert accounting.SWA_BYTES == want["swa_entry_bytes"] == quant.FP8_ENTRY_BYTES
    g4 = accounting.v41_flash_groups(accounting.MAIN_KV_BYTES, accounting.INDEXER_K_BYTES)
    assert accounting.global_bytes_per_token(g4) == want["global_bytes_per_token_fp4"]
    g16 = accounting.v41_flash_groups(512 * 2, 128 * 2)
    assert accounting.global_bytes_per_token(g16) == want["global_bytes_per_token_bf16"]
    r = accounting.retained_bytes(131072, g16, swa_layers=40, swa_bytes=512 * 2, window=128)
    assert r == want["retained_bytes_per_sequence_bf16_131072"]
    assert r // 131072 == want["retained_bytes_per_token_bf16_131072"] and r % 131072 == 0
