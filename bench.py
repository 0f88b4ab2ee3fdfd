"""Benchmark of the CSA2 compressed sparse-attention decode step.

Workload (default): ``hier_1m`` - 4 sequences at a 1,048,576-token FP4 cache,
64 query heads, indexer 8 x 64 FP8, Top-K 2048, window 128; a Full layer that
scores all positions and builds the 2048-block x 8-position candidate pool,
then three Reindex layers that score only the pool.  One step = one decode
token through the whole stack (append-encode of the new token's FP4 / FP8
entries, indexer scores, Top-K, pool, attention) via ``csa_layer_step``.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  Under torchrun every rank runs its own
sequences (replicas, weak scaling) and the step time is the max over ranks.
``--impl reference`` times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import re
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "hier_1m"
METRIC = "decode sparse-attn tokens/s and achieved HBM GB/s vs peak at 1M ctx, FP4 KV"
FLUSH_BYTES = 256 << 20          # > 126 MB L2
L2_BYTES = 126 << 20


def _file_peaks():
    """The machine's measured peaks (context beside the in-run ones), else
    the recipe's fallback figures."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]), "kind": "measured (file)"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "kind": "fallback"}


def _time_ms(fn, reps, stream):
    """Best CUDA-event time of `reps` calls (after two untimed calls)."""
    import torch
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(reps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        best = min(best, a.elapsed_time(b))
    return best


def measure_peaks(dev):
    """The roofline denominators, measured in this run on this GPU:
    * hbm_gbs: the library's 128-bit copy kernel over 2 GiB (read + write);
    * fp8_tflops: the library's tcgen05 FP8 GEMM at 8192^3, cross-checked
      with cuBLAS FP8 (torch._scaled_mm); the larger of the two is the peak;
    * bf16_tflops: cuBLAS bf16 GEMM at 8192^3 (torch.matmul)."""
    import torch
    import indexer_selected_sparse_csa2_b200 as csa
    stream = torch.cuda.current_stream()
    out = {}
    n = 2 << 30
    src = torch.empty(n, dtype=torch.uint8, device=dev)
    dst = torch.empty(n, dtype=torch.uint8, device=dev)
    src.fill_(7)
    ms = _time_ms(lambda: csa.csa_bench_copy(src, dst, stream=stream), 10, stream)
    out["hbm_gbs"] = round(2 * n / (ms * 1e-3) / 1e9, 1)
    out["copy_bytes"] = 2 * n
    del src, dst
    S = 8192
    g = torch.Generator(device=dev).manual_seed(5)
    A = torch.randint(0, 126, (S, S), dtype=torch.uint8, device=dev, generator=g)   # finite E4M3 codes
    B = torch.randint(0, 126, (S, S), dtype=torch.uint8, device=dev, generator=g)
    D = torch.empty(S, S, dtype=torch.float32, device=dev)
    flops = 2.0 * S ** 3
    ms = _time_ms(lambda: csa.csa_bench_fp8_gemm(A, B, D, stream=stream), 5, stream)
    own = flops / (ms * 1e-3) / 1e12
    out["fp8_own_tflops"] = round(own, 1)
    try:
        a8 = A.view(torch.float8_e4m3fn)
        b8 = B.view(torch.float8_e4m3fn)
        one = torch.ones((), dtype=torch.float32, device=dev)
        ms_c = _time_ms(lambda: torch._scaled_mm(a8, b8.t(), scale_a=one, scale_b=one,
                                                 out_dtype=torch.bfloat16), 5, stream)
        out["fp8_cublas_tflops"] = round(flops / (ms_c * 1e-3) / 1e12, 1)
    except Exception as e:       # cross-check only
        out["fp8_cublas_error"] = repr(e)[:120]
    out["fp8_tflops"] = max(out["fp8_own_tflops"], out.get("fp8_cublas_tflops", 0.0))
    del A, B, D
    x = torch.randn(S, S, dtype=torch.bfloat16, device=dev)
    y = torch.randn(S, S, dtype=torch.bfloat16, device=dev)
    ms = _time_ms(lambda: torch.matmul(x, y), 5, stream)
    out["bf16_tflops"] = round(flops / (ms * 1e-3) / 1e12, 1)
    del x, y
    torch.cuda.empty_cache()
    out["kind"] = "measured in this run (burst: kernels timed alone)"
    out["file"] = _file_peaks()
    return out


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest value over all ranks; every rank calls it at the same point
    (a device timing is reported as the slowest rank's)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: the tokens every rank decoded in one step over the
    slowest rank's step time."""
    return tokens_per_rank * world / (ms_max * 1e-3)


def _algorithmic_bytes(cfg):
    """HBM bytes a step must move (indexer keys + selected FP4 entries + window)."""
    per_layer_sel = cfg.B * cfg.K * 288
    per_layer_win = cfg.B * cfg.n_win * 528
    keys = 0
    for L in cfg.layers:
        if L.mode == 2:
            continue
        if L.pool_from >= 0:
            keys += cfg.B * cfg.pool_blocks * cfg.pool_block_len * 64
        else:
            keys += cfg.B * cfg.T * 64
    return keys + len(cfg.layers) * (per_layer_sel + per_layer_win)


KERNEL_SOURCES = {
    "index_score_tc[full]": "index_tc.cu",
    "index_score_mx": "index_mx.cu",
    "index_score_decode[pool]": "index_decode.cu",
    "sparse_attn_tc": "attn_tc.cu",
    "attn_combine": "attn_mma.cu",
    "pool_select": "select_cluster.cu",
    "pool_gather_select": "select_cluster.cu",
    "pool_score_select": "select_cluster.cu",
    "topk_select": "select_cluster.cu",
    "quant_batch": "quant.cu",
    "quant_fp4": "quant.cu",
}


def _traffic_record(kernel):
    """DRAM bytes per launch of `kernel` from a committed ncu summary under
    profiles/ ("bench_kernel: <name>", "traffic_bytes_per_launch: <n>",
    "kernel_source_sha1: <sha>"), only while that kernel's source file still
    has the recorded sha1; else None."""
    import glob
    src = KERNEL_SOURCES.get(kernel)
    if not src:
        return None
    sha = hashlib.sha1(open(os.path.join(ROOT, "indexer_selected_sparse_csa2_b200", "csrc", src), "rb")
                       .read()).hexdigest()
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        txt = open(path).read()
        for blk in txt.split("bench_kernel:")[1:]:
            name = blk.split()[0]
            m = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", blk)
            h = re.search(r"kernel_source_sha1:\s*([0-9a-f]+)", blk)
            if name == kernel and m and h and h.group(1) == sha:
                return int(m.group(1))
    return None


def kernel_work(cfg):
    """Algorithmic HBM bytes and flops per launch of the decode step's kernels
    (what the kernel must read or write, and the multiply-adds x 2 it must do):
    * full scorer: B*T keys of 64 B; 2*64*H_I flops per (key, head);
    * pool select: the B*T/8 block maxima (4 B each) it reads;
    * pool layer score + select: B*pool keys of 64 B (one Reindex layer per launch);
    * the Full layer's select inside its pool: B*pool scores gathered (4 B);
    * attention: B*(K*288 + W*528) entry bytes; 2 * 2*H*512 flops per entry
      (logits and the weighted sum), one layer per launch;
    * split combine: the partial O it reads (B * splits * H * 512 * 4 B)."""
    B, T, K, W, H, HI = cfg.B, cfg.T, cfg.K, cfg.n_win, cfg.H, cfg.H_I
    n_pool = cfg.pool_blocks * cfg.pool_block_len
    nb = (T + cfg.pool_block_len - 1) // cfg.pool_block_len
    return {
        "index_score_tc[full]": {"bytes": B * T * 64, "flops": 2.0 * B * T * HI * 64, "engine": "fp8"},
        "pool_select": {"bytes": B * nb * 4, "flops": 0.0, "engine": None},
        "pool_score_select": {"bytes": B * n_pool * 64, "flops": 2.0 * B * n_pool * HI * 64, "engine": "fp8"},
        "pool_gather_select": {"bytes": B * n_pool * 4, "flops": 0.0, "engine": None},
        "sparse_attn_tc": {"bytes": B * (K * 288 + W * 528), "flops": 4.0 * B * H * 512 * (K + W), "engine": "bf16"},
    }


def roofline_of(name, work, ms_launch, peaks, traffic):
    """Roofline record of one kernel: achieved bytes/s and flops/s against the
    measured HBM and tensor peaks; `bound` is the roof it is nearer to."""
    w = work.get(name)
    if not w or not ms_launch or ms_launch != ms_launch:
        return {"kernel": name, "launch_ms": ms_launch, "bound": None, "achieved": None, "peak": None,
                "unit": None, "frac": None, "traffic": traffic, "note": "no algorithmic work recorded"}
    gbs = w["bytes"] / (ms_launch * 1e-3) / 1e9
    hbm_frac = gbs / peaks["hbm_gbs"]
    rec = {"kernel": name, "launch_ms": round(ms_launch, 5), "bytes_per_launch": w["bytes"],
           "flops_per_launch": w["flops"], "hbm_gbs": round(gbs, 1), "hbm_frac": round(hbm_frac, 4)}
    t_frac = None
    if w["engine"]:
        tpeak = peaks["fp8_tflops"] if w["engine"] == "fp8" else peaks["bf16_tflops"]
        tfl = w["flops"] / (ms_launch * 1e-3) / 1e12
        t_frac = tfl / tpeak
        rec.update({"tflops": round(tfl, 2), "tensor_peak": tpeak, "tensor_frac": round(t_frac, 4),
                    "tensor_peak_kind": f"measured {w['engine']} in this run"})
    if t_frac is not None and t_frac > hbm_frac:
        rec.update({"bound": "tensor", "achieved": rec["tflops"], "peak": rec["tensor_peak"], "unit": "TFLOP/s",
                    "frac": round(t_frac, 4)})
    else:
        rec.update({"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(hbm_frac, 4)})
    rec["traffic"] = traffic
    rec["peak_kind"] = "measured in this run (burst)"
    return rec


class Clocks:
    """SM clock and clock-event reasons sampled by NVML every 2 ms during the
    timed region (read-only queries; no setting is changed)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index):
        self.cuda_index = cuda_index
        self.samples = []
        self.thread = None
        self.stop_flag = False
        self.h = None
        self.err = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(cuda_index).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.nv = pynvml
        except Exception as e:  # no NVML: report no clock record
            self.err = repr(e)
            self.h = None

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_flag:
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM), get_reasons(self.h)))
            except Exception as e:
                self.err = repr(e)
                return
            time.sleep(0.002)

    def start(self):
        if self.h is None:
            return
        import threading
        self.samples = []
        self.stop_flag = False
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def stop(self):
        if self.h is None or self.thread is None:
            return {"error": self.err} if self.err else None
        self.stop_flag = True
        self.thread.join()
        if not self.samples:
            return None
        reasons = set()
        for _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(c for c, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples)}


# --------------------------------------------------------------- reference --
def _oracle_case(cfg):
    """Oracle inputs for sequence 0, prepared outside any timing: encoded keys
    of every owner, the fp32 main latents of every position (the oracle encodes
    the rows a step gathers on demand), each layer's own tensors."""
    from oracle.case import SynthCase
    from oracle import quant as oq
    from csa_synth import workload as wl
    nt = os.cpu_count() or 1
    case = SynthCase(cfg, 0, threads=nt)
    lat = {}
    for o in cfg.owners:
        case.keys(o)
        lat[o] = wl.main_latent(cfg, o, 0, 0, cfg.T, threads=nt)
    case.main_entries = lambda owner, pos: oq.fp4_quant_rows(lat[owner][pos])
    inputs = [case.inputs(li) for li in range(len(cfg.layers))]
    case.inputs = lambda li: inputs[li]
    return case


def _time_oracle(case, n_runs, budget_s=None):
    from threadpoolctl import threadpool_limits
    times = []
    t_end = None if budget_s is None else time.perf_counter() + budget_s
    with threadpool_limits(1):
        while len(times) < n_runs:
            t0 = time.perf_counter()
            case.run()
            times.append(time.perf_counter() - t0)
            if t_end is not None and time.perf_counter() > t_end:
                break
    return times


REF_BUDGET_S = 150.0               # whole --impl reference run
REF_S_PER_POSITION = 5e-6          # oracle cost per cached position (one sequence, all layers), host core


def run_reference(args, cfg, rank, world):
    """The CPU oracle as it stands, on the host cores.  Each step is one
    sequence's decode token through the whole layer stack over a cache of T_s
    positions: T_s = T when (warmup + steps) full steps fit the time budget,
    else the largest power of two that does (the oracle's cost is linear in
    the cache length; the value is scaled back to the full cache)."""
    if rank != 0:
        return
    n = args.steps + args.warmup
    t_s = cfg.T
    while t_s > 65536 and n * t_s * REF_S_PER_POSITION > REF_BUDGET_S:
        t_s //= 2
    scfg = cfg.replace(T=t_s)
    case = _oracle_case(scfg)
    warm = _time_oracle(case, args.warmup)
    slope = 0.0                       # seconds per cache position beyond the sample
    if t_s < cfg.T:
        # per-position cost from a second, half-size cache (untimed, like the warm-up)
        half = _time_oracle(_oracle_case(cfg.replace(T=t_s // 2)), 2)
        slope = max(0.0, (min(warm) - min(half)) / (t_s - t_s // 2))
    times = _time_oracle(case, args.steps)
    ms_sample = 1e3 * sum(times) / len(times)
    ms = ms_sample + 1e3 * slope * (cfg.T - t_s)
    v = 1e3 / ms
    sample = (f"sequence 0 of {WORKLOAD} per step (one decode token, all {len(cfg.layers)} layers)"
              + ("" if t_s == cfg.T else f" over the first {t_s} of {cfg.T} cache positions "
                 f"({ms_sample:.0f} ms per sampled step), extended to the full cache with the per-position "
                 f"cost {slope * 1e9:.0f} ns measured between caches of {t_s // 2} and {t_s} positions"))
    line = {
        "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD, "B_timed": 1, "T": cfg.T, "T_sampled": t_s, "H": cfg.H, "H_I": cfg.H_I,
                   "K": cfg.K, "W": cfg.W, "layers": "Full+pool(2048x8), 3x Reindex-in-pool"},
        "cpu_baseline": {"value": round(v, 4), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": sample, "host": host_cpu()},
        "e2e": {"value": round(v, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def host_cpu():
    """CPU model and logical core count of the host the oracle runs on."""
    model = "unknown"
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"cpu_model": model, "logical_cores": os.cpu_count()}


def cpu_baseline(cfg, seconds_budget=30.0):
    """Oracle timed on one sequence's whole decode step (inputs prepared beforehand)."""
    case = _oracle_case(cfg)
    times = _time_oracle(case, 3, budget_s=seconds_budget)
    s = min(times)
    return {"value": round(1.0 / s, 4), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"sequence 0 of {WORKLOAD}: one decode token through all {len(cfg.layers)} layers "
                      f"(best of {len(times)} runs, {s:.2f} s each; one thread: the oracle as it stands)",
            "host": host_cpu()}


# ---------------------------------------------------------------------- gpu --
def run_gpu(args, cfg, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist
    import indexer_selected_sparse_csa2_b200 as csa
    from csa_synth.device import DeviceCase

    torch.cuda.set_device(local_rank)
    dev = f"cuda:{local_rank}"
    measured_peaks = measure_peaks(dev)
    dc = DeviceCase(cfg, device=dev)
    # per-step inputs and outputs packed into one device buffer each (one
    # host <-> device copy per direction in the end-to-end pass)
    descs = dc.layer_descs(append_rows=True, packed=True)
    ws_bytes = csa.csa_layer_workspace_size(descs)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    # L2 between steps: a step that reads more than the L2 holds evicts the
    # previous step's data by itself; otherwise (or with --flush-l2) a 256 MiB
    # write flushes it, outside the timed events
    do_flush = args.flush_l2 or _algorithmic_bytes(cfg) <= L2_BYTES
    flush_buf = torch.empty(FLUSH_BYTES if do_flush else 16, dtype=torch.uint8, device=dev)

    def flush_l2():
        if do_flush:
            flush_buf.zero_()

    stream = torch.cuda.current_stream()

    def step():
        csa.csa_layer_step(descs, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- device-timed steps
    # The step is captured once into a CUDA graph (as a decode loop runs it);
    # the library's per-kernel events become graph nodes, read after each replay.
    clocks = Clocks(local_rank)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    kernels = {}

    def capture(profile):
        csa.profile_reset()
        csa.profile_enable(profile)
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        n_before = csa.launch_count()
        with torch.cuda.graph(g, stream=cap):
            csa.csa_layer_step(descs, workspace=ws, stream=cap)
        torch.cuda.synchronize()
        csa.profile_enable(False)
        return g, csa.launch_count() - n_before

    def timed(run, ev_start, ev_end, snap):
        for i in range(args.steps):
            flush_l2()
            ev_start[i].record(stream)
            run()
            ev_end[i].record(stream)
            if snap:
                torch.cuda.synchronize()
                for k, (nl, ms_k) in csa.profile_snapshot().items():
                    acc = kernels.setdefault(k, [0, 0.0])
                    acc[0] += nl
                    acc[1] += ms_k
        torch.cuda.synchronize()

    n0 = csa.launch_count()
    if args.no_graph:
        run_step = step
        launches_per_step = None
    else:
        graph, launches_per_step = capture(False)
        run_step = graph.replay
        for _ in range(args.warmup):
            flush_l2()
            run_step()
        torch.cuda.synchronize()
    # 1. headline: the step with no profiling events
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    timed(run_step, starts, ends, False)
    barrier()
    if args.no_graph:
        launches = csa.launch_count() - n0
    else:
        launches = launches_per_step * args.steps
    # 2. per-kernel breakdown (events around every library kernel, same workload)
    p_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    p_ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if args.no_graph:
        csa.profile_enable(True)
        timed(run_step, p_starts, p_ends, False)
        csa.profile_enable(False)
        kernels = {k: list(v) for k, v in csa.profile_collect().items()}
    else:
        pgraph, _ = capture(True)
        for _ in range(2):
            pgraph.replay()
        torch.cuda.synchronize()
        timed(pgraph.replay, p_starts, p_ends, True)
        csa.profile_reset()
    profiled_ms = sum(s_.elapsed_time(e_) for s_, e_ in zip(p_starts, p_ends)) / args.steps
    kernels = {k: (int(v[0]), float(v[1])) for k, v in kernels.items()}
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = sum(step_ms) / len(step_ms)
    ms_max = max_over_ranks(ms, world, dev)

    # ---- end to end through the public call: per-step inputs from pinned host
    # memory, the step, outputs back to pinned host memory
    # The step's inputs: every layer's attention query (dc.step_q), and its
    # index queries, head weights and appended source rows (dc.step_in); its
    # outputs: every layer's out, lse and indices (dc.step_out, layer by
    # layer).  The small inputs go in on the step's stream before the call;
    # the queries on a copy stream that the step waits for only before it
    # first reads them, and each layer's outputs come back on that stream as
    # soon as the layer is done (csa_layer_step_sync's hooks).
    h_in = dc.step_in.cpu().pin_memory()
    h_q = dc.step_q.cpu().pin_memory()
    h_out = torch.empty_like(dc.step_out, device="cpu").pin_memory()
    bi = h_in.numel() + h_q.numel()
    bo = h_out.numel()
    copy_stream = torch.cuda.Stream()
    q_ready = torch.cuda.Event()
    layer_done = [torch.cuda.Event() for _ in cfg.layers]
    for ev in [q_ready] + layer_done:
        ev.record(stream)           # (torch creates an event at its first record)
    torch.cuda.synchronize()

    def step_e2e(i):
        e_starts[i].record(stream)
        dc.step_in.copy_(h_in, non_blocking=True)
        copy_stream.wait_event(e_starts[i])
        with torch.cuda.stream(copy_stream):
            dc.step_q.copy_(h_q, non_blocking=True)
            q_ready.record(copy_stream)
        # the C-ABI call itself, launched eagerly
        csa.csa_layer_step(descs, workspace=ws, stream=stream, queries_ready=q_ready, layer_done=layer_done)
        with torch.cuda.stream(copy_stream):
            for li, (o0, o1) in enumerate(dc.step_out_ranges):
                copy_stream.wait_event(layer_done[li])
                h_out[o0:o1].copy_(dc.step_out[o0:o1], non_blocking=True)
        stream.wait_stream(copy_stream)
        e_ends[i].record(stream)
    e_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for _ in range(2):
        step_e2e(0)                 # warm the eager path (not timed)
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush_l2()
        step_e2e(i)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    if clk is not None and "samples" in clk:
        clk["window"] = "headline, per-kernel and end-to-end passes"
    e2e_ms = sum(s.elapsed_time(e) for s, e in zip(e_starts, e_ends)) / args.steps
    e2e_ms = max_over_ranks(e2e_ms, world, dev)

    if rank != 0:
        return
    peaks = measured_peaks
    hbm_peak = peaks["hbm_gbs"]
    value = job_tokens_per_s(cfg.B, world, ms_max)
    alg = _algorithmic_bytes(cfg)
    # the dominant kernel: the largest share of the step by the per-kernel events
    work = kernel_work(cfg)
    per_step = {k: v[1] / args.steps for k, v in kernels.items()}
    name = max(per_step, key=per_step.get) if per_step else None
    recs = {}
    for k, (nl, tot) in kernels.items():
        if k in work:
            recs[k] = roofline_of(k, work, tot / nl if nl else None, peaks, _traffic_record(k))
    roof = recs.get(name) or roofline_of(name, work, (kernels[name][1] / kernels[name][0]) if name else None,
                                         peaks, None)
    roof["share_of_step"] = round(per_step[name] / max(sum(per_step.values()), 1e-12), 4) if name else None
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8/fp4 storage, fp32 scores, fp16 MMA",
        "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD, "launch": "eager" if args.no_graph else "cuda graph",
                   "B_per_gpu": cfg.B, "T": cfg.T, "H": cfg.H, "H_I": cfg.H_I,
                   "K": cfg.K, "W": cfg.W, "layers": "Full+pool(2048x8), 3x Reindex-in-pool",
                   "parallelism": f"replicas x{world}", "l2": ("flushed between steps (256 MiB write)" if do_flush else
                          f"not flushed: each step reads {_algorithmic_bytes(cfg) / 1e6:.0f} MB > 126 MB L2")},
        "step_hbm_gbs": round(alg / (ms_max * 1e-3) / 1e9, 1),
        "step_hbm_frac": round(alg / (ms_max * 1e-3) / 1e9 / hbm_peak, 4),
        "step_algorithmic_bytes": alg,
        "roofline": roof,
        "roofline_kernels": {k: v for k, v in recs.items() if k != name},
        "peaks": peaks,
        "kernels": {k: {"launches": v[0], "ms_per_step": round(v[1] / args.steps, 5)} for k, v in kernels.items()},
        "kernels_note": f"from a second timed pass with an event pair around every kernel "
                        f"({round(profiled_ms, 4)} ms/step with the events)",
        "gpu_launches": int(launches),
        "e2e": {"value": round(job_tokens_per_s(cfg.B, world, e2e_ms), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": int(bi), "d2h_bytes_per_step": int(bo), "ms_per_step": round(e2e_ms, 4),
                "path": "csa_layer_step_sync called through the Python binding each step (no graph); the "
                        "step's inputs copied in from pinned host memory (index queries, head weights and appended "
                        "rows before the call; the attention queries on a copy stream the step waits for before "
                        "it first reads them) and every layer's out, lse and indices copied back to pinned host "
                        "memory as soon as that layer is done, all inside the timed events"},
        "clocks": clk,
    }
    if world == 1 and not args.no_prefill:
        del dc, descs, ws
        torch.cuda.empty_cache()
        line["prefill"] = run_prefill(args, dev, peaks)
    if world == 1 and not args.no_secondary:
        line["secondary"] = run_secondary(args, dev, peaks)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, seconds_budget=args.cpu_seconds)
    print(json.dumps(line), flush=True)


def _graph_ms(step, reps, stream):
    """Median CUDA-event time of a captured step (replayed `reps` times after 3 warm replays)."""
    import torch
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        step(cap)
    torch.cuda.synchronize()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        b.synchronize()
        ts.append(a.elapsed_time(b))
    del g
    return statistics.median(ts)


def run_secondary(args, dev, peaks):
    """The other rows of the path, timed in this run (not the headline):
    * quant_fp4: the FP4 main-KV encoder over a full 1M-context cache (4 x 2^20
      rows of fp32 latents -> 288-byte entries), GB/s of its reads + writes;
    * decode_mx: one decode step of the pages' MXFP4 indexer shape (8 x 65,536
      positions, 32 heads x 128, top-512), with the MXFP4 scorer's GB/s;
    * ced_40: one decode step of the 40-layer encoder-decoder stack (4 x
      131,072 tokens: 2 SWA, 3 x [Full, 5 Reuse] on one entry per 2 tokens,
      [Full, 3 Reuse] + 4 x [Reindex, 3 Reuse] on the decoder's cache)."""
    import torch
    import indexer_selected_sparse_csa2_b200 as csa
    from csa_synth import get_config
    from csa_synth.device import DeviceCase
    stream = torch.cuda.current_stream()
    out = {}
    # FP4 encoder
    n = 4 << 20
    g = torch.Generator(device=dev).manual_seed(11)
    src = torch.randn((n, 512), dtype=torch.float32, device=dev, generator=g)
    dst = torch.empty((n, 288), dtype=torch.uint8, device=dev)
    ms = _time_ms(lambda: csa.csa_quant_kv(src, csa.CSA_FMT_FP4_E2M1_E4M3X16, dst, stream=stream), 5, stream)
    nbytes = n * (512 * 4 + 288)
    out["quant_fp4"] = {"rows": n, "ms": round(ms, 3), "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                        "hbm_frac": round(nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                        "bytes": nbytes, "note": "fp32 [4M, 512] read + 288-B entries written"}
    del src, dst
    torch.cuda.empty_cache()
    for name in ("decode_mx", "ced_40"):
        cfg = get_config(name)
        dc = DeviceCase(cfg, device=dev)
        descs = dc.layer_descs(append_rows=True)
        ws = torch.empty(max(csa.csa_layer_workspace_size(descs), 16), dtype=torch.uint8, device=dev)
        ms = _graph_ms(lambda st: csa.csa_layer_step(descs, workspace=ws, stream=st), 20, stream)
        rec = {"workload": name, "B": cfg.B, "T": cfg.T, "H_I": cfg.H_I, "d_I": cfg.d_I, "K": cfg.K,
               "layers": len(cfg.layers), "ms_per_step": round(ms, 4),
               "tokens_per_s": round(cfg.B / (ms * 1e-3), 1)}
        if name == "decode_mx":
            # the scorer alone (per-kernel events of one captured step)
            csa.profile_reset()
            csa.profile_enable(True)
            csa.csa_layer_step(descs, workspace=ws, stream=stream)
            torch.cuda.synchronize()
            csa.profile_enable(False)
            kern = csa.profile_collect()
            nl, tot = kern.get("index_score_mx", (0, 0.0))
            if nl:
                kb = cfg.B * cfg.T * 68
                rec["scorer"] = {"kernel": "index_score_mx", "launch_ms": round(tot / nl, 4), "bytes": kb,
                                 "gbs": round(kb / (tot / nl * 1e-3) / 1e9, 1),
                                 "hbm_frac": round(kb / (tot / nl * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                                 "traffic": _traffic_record("index_score_mx"),
                                 "note": "68 B per key (64 code + 4 exponent bytes); one eager launch with events"}
        out[name] = rec
        del dc, descs, ws
        torch.cuda.empty_cache()
    return out


def run_prefill(args, dev, peaks):
    """One prefill chunk (4096 causal queries at a 2^20-token cache): the
    step's FP4 / FP8 encodes of the new tokens, the FP8 tcgen05 indexer GEMM
    with exact per-query Top-K, and attention for every query."""
    import torch
    import indexer_selected_sparse_csa2_b200 as csa
    from csa_synth import get_config
    from csa_synth.device import DeviceCase
    cfg = get_config(args.prefill_config)
    dc = DeviceCase(cfg, device=dev)
    descs = dc.layer_descs(append_rows=True)
    ws = torch.empty(max(csa.csa_layer_workspace_size(descs), 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.prefill_warmup):
        csa.csa_layer_step(descs, workspace=ws, stream=stream)
    torch.cuda.synchronize()
    csa.profile_enable(True)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.prefill_steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.prefill_steps)]
    for i in range(args.prefill_steps):
        starts[i].record(stream)
        csa.csa_layer_step(descs, workspace=ws, stream=stream)
        ends[i].record(stream)
    torch.cuda.synchronize()
    csa.profile_enable(False)
    kern = csa.profile_collect()
    assert csa.device_status() == 0
    ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / args.prefill_steps
    fp8_peak = peaks["fp8_tflops"]
    P = cfg.T - cfg.n_q
    # dense indexer work: n_q x 8 heads x 64 x (keys visible to each query) x 2
    flops = sum(2.0 * cfg.H_I * cfg.d_I * (P + t + 1) for t in range(cfg.n_q))
    nl, tot = kern.get("prefill_score_tc[main]", (0, 0.0))
    main_ms = tot / nl if nl else float("nan")
    tflops = flops / (main_ms * 1e-3) / 1e12 if nl else None
    attn_flops = 2.0 * 2.0 * cfg.n_q * cfg.H * cfg.D * (cfg.K + cfg.n_win)
    return {
        "workload": cfg.name, "n_q": cfg.n_q, "T": cfg.T, "K": cfg.K, "W": cfg.W,
        "ms_per_chunk": round(ms, 3), "tokens_per_s": round(cfg.n_q / (ms * 1e-3), 1),
        "index_gemm": {"bound": "tensor", "achieved": round(tflops, 1) if tflops else None,
                       "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                       "frac": round(tflops / fp8_peak, 4) if tflops else None,
                       "flops_per_launch": flops, "launch_ms": round(main_ms, 4),
                       "peak_kind": "measured fp8 in this run (own tcgen05 GEMM and cuBLAS, the larger)"},
        "attention_tflops": round(attn_flops / (kern.get("sparse_attn_tc", kern.get("sparse_attn_mma", (1, float("nan"))))[1] /
                                                max(1, args.prefill_steps) * 1e-3) / 1e12, 1),
        "kernels": {k: {"launches": v[0], "ms_per_chunk": round(v[1] / args.prefill_steps, 4)}
                    for k, v in kern.items()},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=30.0)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-secondary", action="store_true", help="skip the encoder, decode_mx and ced_40 lines")
    ap.add_argument("--no-graph", action="store_true", help="launch the step eagerly instead of from a CUDA graph")
    ap.add_argument("--flush-l2", action="store_true", help="write 256 MiB between steps even when the step's inputs exceed L2")
    ap.add_argument("--prefill-steps", type=int, default=3)
    ap.add_argument("--prefill-warmup", type=int, default=1)
    ap.add_argument("--prefill-config", default="prefill_1m")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    from csa_synth import get_config
    cfg = get_config(args.workload)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, cfg, rank, world)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_gpu(args, cfg, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
