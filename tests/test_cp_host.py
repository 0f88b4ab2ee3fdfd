"""Host sequencing of the context-parallel decode (indexer_selected_sparse_csa2_b200.context_parallel),
run for real as two gloo ranks on 127.0.0.1 (CPU only).

The per-rank operations here are the oracle's (oracle/context_parallel.py and
the oracle indexer / attention), so the test checks the package's sequencing
of the exchange: shard bounds, rank order of the all-gathers, which rank holds
the window, and the merge / combine inputs.  The device kernels behind the
same operations are checked on a GPU in test_gpu_context_parallel.py.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _OracleShard:
    """The four per-rank operations written with the oracle (float64 / exact),
    exchanging torch CPU tensors."""

    def __init__(self, case, cfg):
        self.case, self.cfg = case, cfg
        self.inp = case.inputs(0)

    def local_topk(self, t0, t1):
        import torch
        from oracle import context_parallel as cpr
        from oracle import indexer as ix
        S = ix.index_scores(self.inp.qI[0], self.inp.w[0], self.case.keys(0)[t0:t1])
        s, p = cpr.local_topk(S, t0, self.cfg.K)
        ps = np.full(self.cfg.K, -np.inf)
        pp = np.full(self.cfg.K, -1, np.int64)
        ps[:s.size], pp[:p.size] = s, p
        return torch.from_numpy(ps)[None], torch.from_numpy(pp)[None]

    def merge(self, gs, gp):
        import torch
        from oracle import context_parallel as cpr
        parts = []
        for r in range(gs.shape[0]):
            keep = gp[r, 0].numpy() >= 0
            parts.append((gs[r, 0].numpy()[keep], gp[r, 0].numpy()[keep]))
        return torch.from_numpy(cpr.merge_topk(parts, self.cfg.K).astype(np.int64))[None]

    def attend(self, idx, t0, t1, with_window):
        import torch
        from oracle import context_parallel as cpr
        from oracle import quant
        sel = idx[0].numpy()
        mine = sel[(sel >= t0) & (sel < t1)].astype(np.int64)
        X = quant.fp4_dequant_rows(self.case.main_entries(0, mine)) if mine.size else np.zeros((0, self.cfg.D))
        if with_window:
            X = np.concatenate([X, quant.fp8_window_dequant_rows(self.inp.window[0:self.cfg.n_win])])
        o, l = cpr.partial_attention(self.inp.q[0], X, self.cfg.softmax_scale)
        return torch.from_numpy(o)[None], torch.from_numpy(l)[None]

    def combine(self, outs, lses):
        import torch
        from oracle import context_parallel as cpr
        o, l = cpr.combine([(outs[r, 0].numpy(), lses[r, 0].numpy()) for r in range(outs.shape[0])])
        return torch.from_numpy(o)[None], torch.from_numpy(l)[None]


def _rank(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from csa_synth import get_config
    from oracle.case import SynthCase
    import importlib.util
    # the host module alone (the package itself loads the CUDA library)
    spec = importlib.util.spec_from_file_location(
        "cp_host", os.path.join(ROOT, "indexer_selected_sparse_csa2_b200", "context_parallel.py"))
    cph = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(cph)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = get_config("tiny_decode", T=3000, K=256)
        ops = _OracleShard(SynthCase(cfg, 0), cfg)
        idx, out, lse = cph.cp_decode(ops, cph.TorchComm(), rank, world, cfg.T)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), idx=idx[0].numpy(), out=out[0].numpy(),
                 lse=lse[0].numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_cp_decode_sequencing_gloo_world2(tmp_path):
    import torch.multiprocessing as mp
    from csa_synth import get_config
    from oracle.case import SynthCase
    mp.spawn(_rank, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    cfg = get_config("tiny_decode", T=3000, K=256)
    ref = SynthCase(cfg, 0).run()[0]
    for r in range(2):
        got = np.load(tmp_path / f"rank{r}.npz")
        assert np.array_equal(got["idx"], ref.idx[0])
        assert np.allclose(got["out"], ref.out[0], rtol=1e-12, atol=1e-13)
        assert np.allclose(got["lse"], ref.lse[0], rtol=1e-12, atol=1e-13)


def test_shard_bounds_match_the_oracle_convention():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "cp_host2", os.path.join(ROOT, "indexer_selected_sparse_csa2_b200", "context_parallel.py"))
    cph = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(cph)
    from oracle import context_parallel as cpr
    for T in (1, 7, 3000, 1 << 20):
        for world in (1, 2, 3, 8):
            assert cph.shard_bounds(T, world) == cpr.shard_bounds(T, world)
