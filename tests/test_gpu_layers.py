"""GPU parity of whole layer stacks (csa_layer_step) vs the oracle.

Small versions of every decode workload; the seeded inputs are encoded on the
device by the library and independently by the oracle.
"""
import numpy as np
import pytest

from csa_synth import get_config
from csa_synth.configs import FULL, REINDEX, REUSE
from oracle.case import SynthCase
from oracle import indexer as oi
from oracle import quant as oq
from tests.parity import topk_diff, assert_close, check_row_format, oracle_attend_on

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def csa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import indexer_selected_sparse_csa2_b200 as m
    return m


def _check_stack(csa, cfg, append=False, sinks=False, batches=None, ws_fill=None):
    from csa_synth.device import DeviceCase
    dc = DeviceCase(cfg, sinks=sinks)
    descs = dc.layer_descs(append_rows=append)
    ws = None
    if ws_fill is not None:
        # a workspace whose every byte is set beforehand (the step must not
        # depend on what it holds)
        ws = torch.full((csa.csa_layer_workspace_size(descs),), ws_fill, dtype=torch.uint8, device="cuda")
        torch.cuda.synchronize()
    csa.csa_layer_step(descs, workspace=ws)
    torch.cuda.synchronize()
    batches = range(cfg.B) if batches is None else batches
    for b in batches:
        case = SynthCase(cfg, b, sinks=sinks)
        res = case.run(keep_scores=True)
        # caches encoded on the device equal the oracle's encodings
        for o in cfg.owners:
            assert np.array_equal(dc.keys[o][b].cpu().numpy(), case.keys(o))
            sample = np.unique(np.concatenate([np.arange(min(cfg.T, 64)), [cfg.T - 1]]))
            assert np.array_equal(dc.kv[o][b, sample].cpu().numpy(), case.main_entries(o, sample))
        for li, L in enumerate(cfg.layers):
            dl = dc.layers[li]
            r = res[li]
            if L.mode == REUSE:
                # no scoring: the step attends over the source layer's indices
                assert np.array_equal(r.idx, res[L.reuse_from].idx)
            else:
                g_idx = dl.idx[b, 0].cpu().numpy()
                check_row_format(g_idx)
                if L.mode == REINDEX and L.pool_from >= 0:
                    P = res[L.pool_from]
                    ppos = P.pool[:P.pool_len].astype(np.int64)
                    S_full = np.full(cfg.T, np.nan)
                    S_full[ppos] = r.scores[0]
                else:
                    S_full = r.scores[0]
                topk_diff(g_idx, r.idx[0], lambda p: S_full[p])
                if L.build_pool:
                    gp = dl.pool[b].cpu().numpy()
                    gn = int(dl.pool_len[b])
                    check_row_format(gp)
                    bm = oi.block_max(r.scores[0], cfg.pool_block_len)
                    gblk = np.unique(gp[:gn] // cfg.pool_block_len)
                    oblk = np.unique(r.pool[:r.pool_len] // cfg.pool_block_len)
                    pad = lambda a: np.concatenate([a, -np.ones(cfg.pool_blocks - a.size, np.int64)])
                    topk_diff(pad(gblk), pad(oblk), lambda p: bm[p])
            # attention on every row: the oracle's result where the index sets
            # agree exactly, else the oracle's attention over the GPU's own set
            src_layer = li if L.mode != REUSE else L.reuse_from
            g_sel = dc.layers[src_layer].idx[b, 0].cpu().numpy()
            if np.array_equal(g_sel, r.idx[0]):
                o_out, o_lse = r.out[0], r.lse[0]
            else:
                o_out, o_lse = oracle_attend_on(case, cfg, li, 0, g_sel)
            assert_close(dl.out[b, 0].cpu().numpy(), o_out, f"layer {li} out")
            assert_close(dl.lse[b, 0].cpu().numpy(), o_lse, f"layer {li} lse")


def test_tiny_decode(csa):
    _check_stack(csa, get_config("tiny_decode"))


def test_tiny_decode_with_append_and_sinks(csa):
    _check_stack(csa, get_config("tiny_decode"), append=True, sinks=True)


def test_decode_outliers_small(csa):
    _check_stack(csa, get_config("decode_64k", B=2, T=20000))


def test_three_layer_stack_small(csa):
    _check_stack(csa, get_config("stack_128k", B=3, T=9001))


def test_hierarchical_small(csa):
    _check_stack(csa, get_config("hier_1m", B=2, T=1 << 16))


def test_hierarchical_ragged_tail(csa):
    _check_stack(csa, get_config("hier_1m", B=1, T=20003, pool_blocks=700, K=300))


def test_cold_first_step(csa):
    """The first step of a fresh process, on a workspace cleared just before
    it: 8 decode tokens with 2 attention tiles per split, where the attention
    epilogue must wait for the PV of the next-to-last tile as well as the last
    (a cold step is where that PV still runs when the softmax warps finish)."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, CSA_COLD_STEP="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", __file__, "-k", "cold_step_body"],
                       env=env, capture_output=True, text=True, cwd=os.path.dirname(os.path.dirname(__file__)))
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


def test_cold_step_body(csa):
    import os
    if os.environ.get("CSA_COLD_STEP") != "1":
        pytest.skip("runs in a fresh process under test_cold_first_step")
    for fill in (0, 255):
        _check_stack(csa, get_config("decode_64k", B=8, T=20000), append=True, ws_fill=fill)


def test_step_sync_hooks_match_plain_step(csa):
    """csa_layer_step_sync: the attention queries uploaded on another stream
    behind a long copy, the step told to wait for them, and every layer's
    outputs downloaded as soon as its layer_done event fires, give the same
    bytes as csa_layer_step with everything resident (4-layer pool stack with
    appends, packed step I/O)."""
    from csa_synth.device import DeviceCase
    cfg = get_config("hier_1m", B=2, T=1 << 15)
    dc = DeviceCase(cfg)
    descs = dc.layer_descs(append_rows=True, packed=True)
    ws = torch.empty(csa.csa_layer_workspace_size(descs), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    csa.csa_layer_step(descs, workspace=ws, stream=stream)
    torch.cuda.synchronize()
    want = dc.step_out.cpu().clone()
    h_q = dc.step_q.cpu().pin_memory()
    h_out = torch.zeros_like(dc.step_out, device="cpu").pin_memory()
    # the queries are destroyed on the device and come back only through the
    # copy stream, after a 256 MiB device copy that delays them
    dc.step_q.zero_()
    dc.step_out.zero_()
    big_a = torch.empty(1 << 28, dtype=torch.uint8, device="cuda")
    big_b = torch.empty_like(big_a)
    torch.cuda.synchronize()
    copy_stream = torch.cuda.Stream()
    q_ready = torch.cuda.Event()
    done = [torch.cuda.Event() for _ in cfg.layers]
    for ev in [q_ready] + done:
        ev.record(stream)
    torch.cuda.synchronize()
    with torch.cuda.stream(copy_stream):
        big_b.copy_(big_a)
        dc.step_q.copy_(h_q, non_blocking=True)
        q_ready.record(copy_stream)
    csa.csa_layer_step(descs, workspace=ws, stream=stream, queries_ready=q_ready, layer_done=done)
    with torch.cuda.stream(copy_stream):
        for li, (o0, o1) in enumerate(dc.step_out_ranges):
            copy_stream.wait_event(done[li])
            h_out[o0:o1].copy_(dc.step_out[o0:o1], non_blocking=True)
    torch.cuda.synchronize()
    for li, (o0, o1) in enumerate(dc.step_out_ranges):
        assert torch.equal(h_out[o0:o1], want[o0:o1]), f"layer {li}"
