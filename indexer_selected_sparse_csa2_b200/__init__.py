"""Python binding of the CSA2 sparse-attention step library (``libcsa.so``).

Argument marshalling only: every step runs in the library's CUDA kernels.
PyTorch provides device memory and streams.  There is no CPU fallback: if the
library is missing, importing this package raises.

The entry points mirror ``include/csa.h``:

* ``csa_quant_kv``       - FP4 / FP8 cache-entry encoding (and plain E4M3 casts)
* ``csa_index_topk``     - lightning-indexer scores + Top-K (+ candidate pool)
* ``csa_topk_scores``    - Top-K of given fp32 scores
* ``csa_sparse_attn``    - sparse MLA attention over selected entries + window
* ``csa_layer_step``     - a Full / Reindex / Reuse layer stack
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python indexer_selected_sparse_csa2_b200/build.py` "
        "(there is no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

# --------------------------------------------------------------- constants --
CSA_OK, CSA_ERR_INVALID_ARG, CSA_ERR_SHAPE, CSA_ERR_ALIGNMENT, CSA_ERR_UNSUPPORTED, \
    CSA_ERR_WORKSPACE, CSA_ERR_CUDA = range(7)
CSA_SRC_F32, CSA_SRC_BF16 = 0, 1
CSA_FMT_FP4_E2M1_E4M3X16, CSA_FMT_FP8_E4M3_UE8M0X32, CSA_FMT_FP8_E4M3_PLAIN = 0, 1, 2
CSA_MODE_FULL, CSA_MODE_REINDEX, CSA_MODE_REUSE, CSA_MODE_SWA = 0, 1, 2, 3
CSA_KEY_E4M3, CSA_KEY_MXFP4 = 0, 1
FP4_ENTRY_BYTES, FP8_ENTRY_BYTES = 288, 528

_p = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_f32 = ctypes.c_float


class IndexArgs(ctypes.Structure):
    _fields_ = [("B", _i32), ("n_q", _i32), ("T", _i64), ("H_I", _i32), ("d_I", _i32),
                ("keys", _p), ("key_row_stride", _i64), ("key_batch_stride", _i64),
                ("q", _p), ("w", _p), ("K", _i32),
                ("pool", _p), ("pool_len", _p), ("pool_cap", _i32),
                ("pool_out", _p), ("pool_out_len", _p), ("pool_blocks", _i32), ("pool_block_len", _i32),
                ("idx", _p), ("scores", _p),
                ("key_format", _i32), ("key_scales", _p), ("key_scale_row_stride", _i64),
                ("key_scale_batch_stride", _i64)]


class AttnArgs(ctypes.Structure):
    _fields_ = [("B", _i32), ("n_q", _i32), ("H", _i32), ("D", _i32),
                ("q", _p), ("kv", _p), ("kv_row_stride", _i64), ("kv_batch_stride", _i64),
                ("idx", _p), ("K", _i32),
                ("win", _p), ("win_row_stride", _i64), ("win_batch_stride", _i64), ("n_win", _i32),
                ("softmax_scale", _f32), ("sink", _p), ("out", _p), ("lse", _p),
                ("rope_cs", _p), ("out_bf16", _i32)]


class QuantJob(ctypes.Structure):
    _fields_ = [("src", _p), ("src_dtype", _i32), ("dim", _i32), ("n_rows", _i64),
                ("src_row_stride", _i64), ("fmt", _i32), ("dst", _p), ("dst_row_stride", _i64)]


class LayerDesc(ctypes.Structure):
    _fields_ = [("mode", _i32), ("reuse_from", _i32), ("pool_from", _i32),
                ("append", QuantJob * 3), ("index", IndexArgs), ("attn", AttnArgs)]


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 56), ("launches", ctypes.c_uint64), ("total_ms", ctypes.c_double)]


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_quant = _sig("csa_quant_kv", _i32, [_p, _i32, _i64, _i32, _i64, _i32, _p, _i64, _p])
_quant_mx = _sig("csa_quant_mxfp4", _i32, [_p, _i32, _i64, _i32, _i64, _p, _i64, _p, _i64, _p])
_compress = _sig("csa_compress_kv", _i32, [_p, _i32, _p, _i64, _i32, _i32, _i64, _i64, _i32, _p, _i64, _p])
_index_ws = _sig("csa_index_workspace_size", ctypes.c_size_t, [ctypes.POINTER(IndexArgs)])
_index = _sig("csa_index_topk", _i32, [ctypes.POINTER(IndexArgs), _p, ctypes.c_size_t, _p])
_index_noalloc = _sig("csa_index_topk_noalloc", _i32, [ctypes.POINTER(IndexArgs), _p])
_index_noalloc_cap = _sig("csa_index_noalloc_capacity", ctypes.c_size_t, [])
_topk_ws = _sig("csa_topk_workspace_size", ctypes.c_size_t, [_i32, _i64])
_topk = _sig("csa_topk_scores", _i32, [_p, _i32, _i64, _i64, _i32, _p, _p, ctypes.c_size_t, _p])
_attn_ws = _sig("csa_attn_workspace_size", ctypes.c_size_t, [ctypes.POINTER(AttnArgs)])
_attn = _sig("csa_sparse_attn", _i32, [ctypes.POINTER(AttnArgs), _p, ctypes.c_size_t, _p])
_layer_ws = _sig("csa_layer_workspace_size", ctypes.c_size_t, [ctypes.POINTER(LayerDesc), _i32])
_layer = _sig("csa_layer_step", _i32, [ctypes.POINTER(LayerDesc), _i32, _p, ctypes.c_size_t, _p])


class StepSync(ctypes.Structure):
    _fields_ = [("queries_ready", _p), ("layer_done", _p * 64)]


_layer_sync = _sig("csa_layer_step_sync", _i32,
                   [ctypes.POINTER(LayerDesc), _i32, _p, ctypes.c_size_t, ctypes.POINTER(StepSync), _p])
_status_string = _sig("csa_status_string", ctypes.c_char_p, [_i32])
_launch_count = _sig("csa_launch_count", ctypes.c_uint64, [])
_device_status = _sig("csa_device_status", _i32, [])
_version = _sig("csa_version", _i32, [])
_profile_enable = _sig("csa_profile_enable", _i32, [_i32])
_profile_collect = _sig("csa_profile_collect", _i32, [ctypes.POINTER(KernelTime), _i32])
_profile_snapshot = _sig("csa_profile_snapshot", _i32, [ctypes.POINTER(KernelTime), _i32])
_profile_reset = _sig("csa_profile_reset", None, [])
_bench_copy = _sig("csa_bench_copy", _i32, [_p, _p, ctypes.c_size_t, _p])
_bench_fp8_gemm = _sig("csa_bench_fp8_gemm", _i32, [_p, _p, _p, _i32, _i32, _i32, _p])
_cp_pairs = _sig("csa_cp_local_pairs", _i32, [_p, _p, _i32, _i32, _i64, _i64, _p, _p, _p])
_cp_merge_ws = _sig("csa_cp_merge_workspace_size", ctypes.c_size_t, [_i32, _i32, _i32])
_cp_merge = _sig("csa_cp_merge_topk", _i32, [_p, _p, _i32, _i32, _i32, _i32, _p, _p, ctypes.c_size_t, _p])
_cp_localize = _sig("csa_cp_localize", _i32, [_p, _i32, _i32, _i64, _i64, _p, _p])
_cp_combine = _sig("csa_cp_combine", _i32, [_p, _p, _i32, _i32, _i32, _p, _p, _p, _p])

EXPORTED = ["csa_quant_kv", "csa_compress_kv", "csa_quant_mxfp4", "csa_index_workspace_size", "csa_index_topk", "csa_topk_workspace_size",
            "csa_topk_scores", "csa_attn_workspace_size", "csa_sparse_attn", "csa_layer_workspace_size",
            "csa_layer_step", "csa_status_string", "csa_launch_count", "csa_version",
            "csa_profile_enable", "csa_profile_collect", "csa_index_topk_noalloc", "csa_device_status",
            "csa_index_noalloc_capacity", "csa_profile_snapshot", "csa_profile_reset",
            "csa_bench_copy", "csa_bench_fp8_gemm", "csa_cp_local_pairs", "csa_cp_merge_workspace_size",
            "csa_cp_merge_topk", "csa_cp_localize", "csa_cp_combine", "csa_layer_step_sync"]


def profile_enable(on: bool) -> bool:
    """Bracket every library kernel launch with CUDA events (see csa.h)."""
    return bool(_profile_enable(1 if on else 0))


def profile_collect() -> dict:
    """{kernel name: (launches, total milliseconds)} since the last collect."""
    buf = (KernelTime * 128)()
    n = _profile_collect(buf, 128)
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms)) for i in range(min(n, 128))}


def profile_snapshot() -> dict:
    """As profile_collect, but keeps the records (graph replays re-record them)."""
    buf = (KernelTime * 128)()
    n = _profile_snapshot(buf, 128)
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms)) for i in range(min(n, 128))}


def profile_reset() -> None:
    _profile_reset()


class CsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


def status_string(status: int) -> str:
    return _status_string(status).decode()


def launch_count() -> int:
    return int(_launch_count())


def device_status() -> int:
    """Error code of a timed-out device wait since the last call (0 = none)."""
    return int(_device_status())


def version() -> int:
    return int(_version())


def _check(status: int, where: str):
    if status != CSA_OK:
        raise CsaError(status, where)


# ------------------------------------------------------------ torch glue --
def _torch():
    import torch
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _workspace(nbytes: int, device):
    torch = _torch()
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


# ------------------------------------------------------------ entry points --
def csa_quant_kv(src, fmt: int, dst, n_rows: Optional[int] = None, dim: Optional[int] = None,
                 src_row_stride: Optional[int] = None, dst_row_stride: Optional[int] = None,
                 stream=None) -> None:
    """Encode rows of ``src`` (fp32 or bf16, [n_rows, dim]) into ``dst`` (uint8)."""
    torch = _torch()
    dtype = CSA_SRC_BF16 if src.dtype == torch.bfloat16 else CSA_SRC_F32
    if src.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("src must be float32 or bfloat16")
    n_rows = src.shape[0] if n_rows is None else n_rows
    dim = src.shape[-1] if dim is None else dim
    src_row_stride = src.stride(0) if src_row_stride is None else src_row_stride
    dst_row_stride = dst.stride(0) * dst.element_size() if dst_row_stride is None else dst_row_stride
    _check(_quant(_ptr(src), dtype, n_rows, dim, src_row_stride, fmt, _ptr(dst), dst_row_stride,
                  _stream(stream)), "csa_quant_kv")


def csa_quant_mxfp4(src, codes, scales, stream=None) -> None:
    """MXFP4 encoding of ``src`` (fp32 / bf16 [n_rows, dim]) into ``codes``
    (uint8 [n_rows, dim/2]) and ``scales`` (uint8 [n_rows, dim/32])."""
    torch = _torch()
    dtype = CSA_SRC_BF16 if src.dtype == torch.bfloat16 else CSA_SRC_F32
    _check(_quant_mx(_ptr(src), dtype, src.shape[0], src.shape[-1], src.stride(0), _ptr(codes),
                     codes.stride(0) * codes.element_size(), _ptr(scales), scales.stride(0) * scales.element_size(),
                     _stream(stream)), "csa_quant_mxfp4")


def csa_compress_kv(src, gate, m: int, fmt: int, dst, dst_row_stride: Optional[int] = None, stream=None) -> None:
    """Pool groups of m token rows of ``src`` (fp32 / bf16 [n_groups * m, dim])
    with the fp32 gate logits ``gate`` ([n_groups * m, dim], None when m == 1)
    and encode each pooled entry into ``dst`` (uint8 rows)."""
    torch = _torch()
    dtype = CSA_SRC_BF16 if src.dtype == torch.bfloat16 else CSA_SRC_F32
    n_groups = src.shape[0] // m
    dim = src.shape[-1]
    dst_row_stride = dst.stride(0) * dst.element_size() if dst_row_stride is None else dst_row_stride
    _check(_compress(_ptr(src), dtype, _ptr(gate), n_groups, m, dim, src.stride(0),
                     0 if gate is None else gate.stride(0), fmt, _ptr(dst), dst_row_stride, _stream(stream)),
           "csa_compress_kv")


def csa_index_workspace_size(args: IndexArgs) -> int:
    return int(_index_ws(ctypes.byref(args)))


def csa_index_topk(args: IndexArgs, workspace=None, stream=None, device=None) -> None:
    need = csa_index_workspace_size(args)
    if workspace is None:
        workspace = _workspace(need, device or "cuda")
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_index(ctypes.byref(args), _ptr(workspace), nbytes, _stream(stream)), "csa_index_topk")


def csa_index_noalloc_capacity() -> int:
    return int(_index_noalloc_cap())


def csa_index_topk_noalloc(args: IndexArgs, stream=None) -> None:
    """csa_index_topk with the library's fixed device scratch instead of a
    caller workspace (see csa.h): for callers that cannot allocate."""
    _check(_index_noalloc(ctypes.byref(args), _stream(stream)), "csa_index_topk_noalloc")


def csa_topk_workspace_size(B: int, n: int) -> int:
    return int(_topk_ws(B, n))


def csa_topk_scores(scores, K: int, idx, workspace=None, stream=None) -> None:
    """Top-K of fp32 ``scores`` [B, n] (row stride from the tensor) into int32 ``idx`` [B, K]."""
    B, n = scores.shape
    if workspace is None:
        workspace = _workspace(csa_topk_workspace_size(B, n), scores.device)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_topk(_ptr(scores), B, n, scores.stride(0), K, _ptr(idx), _ptr(workspace), nbytes,
                 _stream(stream)), "csa_topk_scores")


def csa_attn_workspace_size(args: AttnArgs) -> int:
    return int(_attn_ws(ctypes.byref(args)))


def csa_sparse_attn(args: AttnArgs, workspace=None, stream=None, device=None) -> None:
    # the library checks a given workspace's size itself; query it only to allocate one
    if workspace is None:
        workspace = _workspace(csa_attn_workspace_size(args), device or "cuda")
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_attn(ctypes.byref(args), _ptr(workspace), nbytes, _stream(stream)), "csa_sparse_attn")


def make_layer_array(layers: Sequence[LayerDesc]):
    """ctypes array of LayerDesc.  Assigning an IndexArgs / AttnArgs /
    QuantJob into a LayerDesc copies raw pointers only: the caller keeps the
    tensors they point at alive (attach them to the LayerDesc as `_keep`)."""
    arr = (LayerDesc * len(layers))()
    for i, L in enumerate(layers):
        arr[i] = L
    arr._keep = list(layers)
    return arr


def csa_layer_workspace_size(layers) -> int:
    return int(_layer_ws(layers, len(layers)))


def _event(ev) -> Optional[int]:
    if ev is None:
        return None
    return ev.cuda_event if hasattr(ev, "cuda_event") else int(ev)


def csa_layer_step(layers, workspace=None, stream=None, device=None, queries_ready=None, layer_done=None) -> None:
    """Run a ctypes array of LayerDesc (see ``make_layer_array``) on one stream.
    ``queries_ready`` (a torch.cuda.Event) and ``layer_done`` (one event or
    None per layer) select csa_layer_step_sync: the step reads the attention
    queries only after ``queries_ready`` and records ``layer_done[i]`` once
    layer i's outputs are written."""
    # the library checks a given workspace's size itself; query it only to allocate one
    if workspace is None:
        workspace = _workspace(csa_layer_workspace_size(layers), device or "cuda")
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if queries_ready is None and layer_done is None:
        _check(_layer(layers, len(layers), _ptr(workspace), nbytes, _stream(stream)), "csa_layer_step")
        return
    sync = StepSync()
    sync.queries_ready = _event(queries_ready)
    for i, ev in enumerate(layer_done or []):
        sync.layer_done[i] = _event(ev)
    _check(_layer_sync(layers, len(layers), _ptr(workspace), nbytes, ctypes.byref(sync), _stream(stream)),
           "csa_layer_step_sync")


def csa_bench_copy(src, dst, stream=None) -> None:
    """128-bit copy of ``src`` into ``dst`` (same byte size) by the library's
    copy kernel (the in-run HBM peak)."""
    nbytes = src.numel() * src.element_size()
    assert dst.numel() * dst.element_size() >= nbytes
    _check(_bench_copy(_ptr(src), _ptr(dst), nbytes, _stream(stream)), "csa_bench_copy")


def csa_bench_fp8_gemm(A, B, D, stream=None) -> None:
    """D (fp32 [M, N]) = A (E4M3 bytes [M, K]) x B (E4M3 bytes [N, K])^T on the
    library's tcgen05 FP8 GEMM (the in-run FP8 dense peak)."""
    M, K = A.shape
    N = B.shape[0]
    _check(_bench_fp8_gemm(_ptr(A), _ptr(B), _ptr(D), M, N, K, _stream(stream)), "csa_bench_fp8_gemm")


def csa_cp_local_pairs(idx, scores, t0: int, pair_score, pair_pos, stream=None) -> None:
    """Shard-local Top-K (idx [B, K] or [B, 1, K]) -> (score, global position) pairs."""
    B, K = idx.shape[0], idx.shape[-1]
    _check(_cp_pairs(_ptr(idx), _ptr(scores), B, K, scores.stride(0), t0, _ptr(pair_score), _ptr(pair_pos),
                     _stream(stream)), "csa_cp_local_pairs")


def csa_cp_merge_topk(pair_score, pair_pos, K: int, idx, workspace=None, stream=None) -> None:
    """Gathered pairs [R, B, K_local] (rank order) -> global Top-K idx [B, K]."""
    R, B, Kl = pair_score.shape
    if workspace is None:
        workspace = _workspace(int(_cp_merge_ws(R, B, Kl)), pair_score.device)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_cp_merge(_ptr(pair_score), _ptr(pair_pos), R, B, Kl, K, _ptr(idx), _ptr(workspace), nbytes,
                     _stream(stream)), "csa_cp_merge_topk")


def csa_cp_localize(idx, t0: int, t1: int, idx_local, stream=None) -> None:
    B, K = idx.shape[0], idx.shape[-1]
    _check(_cp_localize(_ptr(idx), B, K, t0, t1, _ptr(idx_local), _stream(stream)), "csa_cp_localize")


def csa_cp_combine(o_parts, lse_parts, out, lse=None, sink=None, stream=None) -> None:
    """o_parts [R, B, H, 512], lse_parts [R, B, H] -> out [B, H, 512], lse [B, H]."""
    R, B, H = lse_parts.shape
    _check(_cp_combine(_ptr(o_parts), _ptr(lse_parts), R, B, H, _ptr(sink), _ptr(out), _ptr(lse),
                       _stream(stream)), "csa_cp_combine")


# ------------------------------------------------------- argument builders --
def index_args(*, keys, q, w, K: int, idx, T: Optional[int] = None, n_q: int = 1,
               pool=None, pool_len=None, pool_out=None, pool_out_len=None,
               pool_blocks: int = 2048, pool_block_len: int = 8, scores=None, key_scales=None) -> IndexArgs:
    """IndexArgs from torch tensors: keys uint8 [B, T, 64] (any row / batch stride),
    q uint8 [B, n_q, H_I, d_I], w fp32 [B, n_q, H_I], idx int32 [B, n_q, K].
    With key_scales (uint8 [B, T, 4]) the keys are MXFP4 codes (d_I = 128)."""
    B = keys.shape[0]
    a = IndexArgs()
    a.B, a.n_q = B, n_q
    a.T = keys.shape[1] if T is None else T
    a.H_I, a.d_I = q.shape[-2], q.shape[-1]
    a.keys, a.key_row_stride, a.key_batch_stride = _ptr(keys), keys.stride(1), keys.stride(0)
    a.q, a.w, a.K = _ptr(q), _ptr(w), K
    if pool is not None:
        a.pool, a.pool_len, a.pool_cap = _ptr(pool), _ptr(pool_len), pool.shape[-1]
    if pool_out is not None:
        a.pool_out, a.pool_out_len = _ptr(pool_out), _ptr(pool_out_len)
    a.pool_blocks, a.pool_block_len = pool_blocks, pool_block_len
    a.idx = _ptr(idx)
    a.scores = _ptr(scores)
    if key_scales is not None:
        a.key_format = CSA_KEY_MXFP4
        a.key_scales = _ptr(key_scales)
        a.key_scale_row_stride, a.key_scale_batch_stride = key_scales.stride(1), key_scales.stride(0)
    # the struct holds raw device pointers: keep the tensors alive with it
    a._keep = (keys, q, w, pool, pool_len, pool_out, pool_out_len, idx, scores, key_scales)
    return a


def attn_args(*, q, kv, idx, win, n_win: int, softmax_scale: float, out, lse=None, sink=None,
              K: Optional[int] = None, rope_cs=None) -> AttnArgs:
    """AttnArgs from torch tensors: q fp32 [B, n_q, H, 512], kv uint8 [B, T, 288],
    idx int32 [B, n_q, K], win uint8 [B, rows, 528], out fp32 or bf16
    [B, n_q, H, 512]; rope_cs optional fp32 [B, n_q, 32, 2] (cos, sin) of each
    query position's angles (partial RoPE on q, inverse rotation on out)."""
    a = AttnArgs()
    a.B, a.n_q, a.H, a.D = q.shape
    a.q = _ptr(q)
    if kv is not None:
        a.kv, a.kv_row_stride, a.kv_batch_stride = _ptr(kv), kv.stride(1), kv.stride(0)
    a.idx = _ptr(idx)
    a.K = idx.shape[-1] if (K is None and idx is not None) else (K or 0)
    if win is not None:
        a.win, a.win_row_stride, a.win_batch_stride = _ptr(win), win.stride(1), win.stride(0)
    a.n_win = n_win
    a.softmax_scale = softmax_scale
    a.sink, a.out, a.lse = _ptr(sink), _ptr(out), _ptr(lse)
    a.rope_cs = _ptr(rope_cs)
    a.out_bf16 = 1 if str(out.dtype) == "torch.bfloat16" else 0
    a._keep = (q, kv, idx, win, out, lse, sink, rope_cs)
    return a


def quant_job(src, fmt: int, dst, dst_row_stride: int, n_rows: Optional[int] = None) -> QuantJob:
    torch = _torch()
    j = QuantJob()
    j.src = _ptr(src)
    j.src_dtype = CSA_SRC_BF16 if src.dtype == torch.bfloat16 else CSA_SRC_F32
    j.dim = src.shape[-1]
    j.n_rows = src.shape[0] if n_rows is None else n_rows
    j.src_row_stride = src.stride(0)
    j.fmt = fmt
    j.dst = _ptr(dst)
    j.dst_row_stride = dst_row_stride
    j._keep = (src, dst)
    return j
