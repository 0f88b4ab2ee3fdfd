"""Full-size GPU parity: every workload at its real size, run exactly as the
benchmark runs it (csa_layer_step over the device-encoded caches, with the
step's new-token encodes), checked against the oracle on sampled sequences
(decode) or sampled query tokens (prefill)."""
import os

import numpy as np
import pytest

from csa_synth import get_config
from csa_synth.configs import FULL, REINDEX, REUSE
from oracle.case import SynthCase
from oracle import indexer as oi
from tests.parity import topk_diff, assert_close, check_row_format, oracle_attend_on

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import indexer_selected_sparse_csa2_b200 as m
    return m


def _compare_layers(cfg, dc, b, res, queries, case):
    """res: oracle results of ``case`` (sequence b) for the query tokens
    ``queries``.  Index sets by the Top-K rule; attention on every row: against
    the oracle's result where the sets agree, else against the oracle's
    attention over the GPU's own index set."""
    n_identical = n_rows = 0
    inputs = {}
    for li, L in enumerate(cfg.layers):
        dl = dc.layers[li]
        r = res[li]
        for qr, t in enumerate(queries):
            n_rows += 1
            if L.mode == REUSE:
                src = L.reuse_from
                g_idx = dc.layers[src].idx[b, t].cpu().numpy()
                o_idx = r.idx[qr]
            else:
                g_idx = dl.idx[b, t].cpu().numpy()
                o_idx = r.idx[qr]
                check_row_format(g_idx)
                if L.mode == REINDEX and L.pool_from >= 0:
                    P = res[L.pool_from]
                    S_full = np.full(cfg.T, np.nan)
                    S_full[P.pool[:P.pool_len].astype(np.int64)] = r.scores[qr]
                else:
                    S_full = r.scores[qr]
                topk_diff(g_idx, o_idx, lambda p: S_full[p])
                if L.build_pool:
                    gp = dl.pool[b].cpu().numpy()
                    gn = int(dl.pool_len[b])
                    check_row_format(gp)
                    bm = oi.block_max(r.scores[qr], cfg.pool_block_len)
                    gblk = np.unique(gp[:gn] // cfg.pool_block_len)
                    oblk = np.unique(r.pool[:r.pool_len] // cfg.pool_block_len)
                    pad = lambda a: np.concatenate([a, -np.ones(cfg.pool_blocks - a.size, np.int64)])
                    topk_diff(pad(gblk), pad(oblk), lambda p: bm[p])
            if np.array_equal(g_idx, o_idx):
                n_identical += 1
                o_out, o_lse = r.out[qr], r.lse[qr]
            else:
                if li not in inputs:
                    inputs[li] = case.inputs(li)
                o_out, o_lse = oracle_attend_on(case, cfg, li, t, g_idx, inputs[li])
            assert_close(dl.out[b, t].cpu().numpy(), o_out, f"layer {li} b {b} t {t} out")
            assert_close(dl.lse[b, t].cpu().numpy(), o_lse, f"layer {li} b {b} t {t} lse")
    # near-tie swaps are allowed by the Top-K rule but must stay rare
    assert n_identical >= 0.75 * n_rows, (n_identical, n_rows)


def _clear_outputs(dc):
    for dl in dc.layers:
        dl.out.zero_()
        dl.lse.zero_()
        dl.idx.fill_(-7)
        if dl.pool is not None:
            dl.pool.fill_(-7)
            dl.pool_len.zero_()


def _run_decode(csa, name, batches, graph=False):
    """The step eagerly; with `graph`, then also captured into a CUDA graph on
    a side stream and replayed, as the benchmark times it (outputs cleared
    before the replay), both checked against the same oracle results."""
    from csa_synth.device import DeviceCase
    cfg = get_config(name)
    dc = DeviceCase(cfg, keep_scores=False)
    descs = dc.layer_descs(append_rows=True)
    ws = torch.empty(max(csa.csa_layer_workspace_size(descs), 16), dtype=torch.uint8, device="cuda")
    csa.csa_layer_step(descs, workspace=ws)
    torch.cuda.synchronize()
    assert csa.device_status() == 0
    results, cases = {}, {}
    for b in batches:
        case = SynthCase(cfg, b, threads=os.cpu_count() or 4, dense_latents=True)
        for o in cfg.owners:
            rows = np.array([0, 1, cfg.T // 2, cfg.T - 1])
            assert np.array_equal(dc.keys[o][b].cpu().numpy()[rows], case.keys(o)[rows])
            assert np.array_equal(dc.kv[o][b, torch.from_numpy(rows)].cpu().numpy(), case.main_entries(o, rows))
        results[b] = case.run(keep_scores=True)
        cases[b] = case
        _compare_layers(cfg, dc, b, results[b], [0], cases[b])
    if graph:
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(g, stream=cap):
            csa.csa_layer_step(descs, workspace=ws, stream=cap)
        torch.cuda.synchronize()
        _clear_outputs(dc)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        assert csa.device_status() == 0
        for b in batches:
            _compare_layers(cfg, dc, b, results[b], [0], cases[b])
        del g


def test_fullsize_tiny_decode(csa):
    _run_decode(csa, "tiny_decode", [0])


def test_fullsize_decode_64k(csa):
    _run_decode(csa, "decode_64k", [0, 7])


def test_fullsize_stack_128k(csa):
    _run_decode(csa, "stack_128k", [0, 31])


def test_fullsize_hier_1m(csa):
    _run_decode(csa, "hier_1m", [0, 3], graph=True)


def test_fullsize_prefill_1m(csa):
    from csa_synth.device import DeviceCase
    cfg = get_config("prefill_1m")
    dc = DeviceCase(cfg)
    csa.csa_layer_step(dc.layer_descs(append_rows=True))
    torch.cuda.synchronize()
    assert csa.device_status() == 0
    qs = [0, 1, 2047, 4095]
    case = SynthCase(cfg, 0, threads=os.cpu_count() or 4, dense_latents=True)
    res = case.run(queries=qs, keep_scores=True)
    _compare_layers(cfg, dc, 0, res, qs, case)
