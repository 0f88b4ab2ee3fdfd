"""Host logic of bench.py's multi-process path on CPU: two ranks over gloo.

bench.py runs one process per GPU (replicas of the decode step, no data-path
collective).  What crosses ranks is the reported timing, which is the slowest
rank's, and the whole-job throughput built from it.  The reference arm runs on
rank 0 alone.  These tests run that logic as two gloo ranks on 127.0.0.1.
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # each rank's own step time; the reported one is the largest
        step_ms = [0.25, 0.75][rank]
        ms_max = bench.max_over_ranks(step_ms, world, "cpu")
        e2e_max = bench.max_over_ranks([0.9, 0.4][rank], world, "cpu")
        value = bench.job_tokens_per_s(4, world, ms_max)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms_max": ms_max, "e2e_max": e2e_max, "value": value}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_world2(tmp_path):
    import torch.multiprocessing as mp
    mp.spawn(_rank_main, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        d = json.load(open(tmp_path / f"rank{r}.json"))
        assert d["ms_max"] == 0.75            # the slower rank's step time, on every rank
        assert d["e2e_max"] == 0.9
        # 2 ranks x 4 sequences, one token each, in 0.75 ms
        assert d["value"] == pytest.approx(8 / 0.75e-3)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.5, 1, "cpu") == 0.5
    assert bench.job_tokens_per_s(4, 1, 0.5) == pytest.approx(8000.0)


def test_reference_arm_runs_on_rank0_only():
    """A rank other than 0 exits 0 at once with no output and no oracle work."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
