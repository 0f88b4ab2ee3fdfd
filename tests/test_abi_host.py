"""C-ABI checks that need no GPU: the library loads, exports every function
declared in include/csa.h, and host-side argument validation rejects bad
arguments before any CUDA call (no kernel is launched by these tests)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(csa_\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def csa():
    import __graft_entry__
    __graft_entry__.build()
    import indexer_selected_sparse_csa2_b200 as m
    return m


def test_every_declared_symbol_is_exported(csa):
    lib = ctypes.CDLL(csa.LIB_PATH)
    declared = _declared()
    assert declared, "no declarations found"
    missing = [n for n in sorted(declared) if not hasattr(lib, n)]
    assert not missing, missing
    assert set(csa.EXPORTED) <= declared


def test_status_strings(csa):
    assert csa.status_string(0) == "ok"
    assert "workspace" in csa.status_string(csa.CSA_ERR_WORKSPACE)
    assert csa.version() >= 1


def test_quant_rejects_bad_args_on_host(csa):
    q = csa._quant
    buf = ctypes.create_string_buffer(4096 + 16)
    addr = (ctypes.addressof(buf) + 15) & ~15
    # NULL source
    assert q(None, 0, 4, 512, 512, 0, addr, 288, None) == csa.CSA_ERR_INVALID_ARG
    # wrong dim for FP4
    assert q(addr, 0, 1, 256, 256, 0, addr, 288, None) == csa.CSA_ERR_SHAPE
    # unknown format
    assert q(addr, 0, 1, 512, 512, 9, addr, 288, None) == csa.CSA_ERR_INVALID_ARG
    # misaligned destination
    assert q(addr, 0, 2, 512, 512, 0, addr + 1, 288, None) == csa.CSA_ERR_ALIGNMENT
    # destination row stride too small
    assert q(addr, 0, 2, 512, 512, 1, addr, 288, None) == csa.CSA_ERR_SHAPE
    # plain cast dim not a multiple of 16
    assert q(addr, 0, 1, 40, 40, 2, addr, 48, None) == csa.CSA_ERR_SHAPE
    # zero rows is a no-op that succeeds without touching the device
    assert q(None, 0, 0, 512, 512, 0, None, 288, None) == csa.CSA_OK


def test_index_rejects_bad_args_on_host(csa):
    a = csa.IndexArgs()
    a.B, a.n_q, a.T, a.H_I, a.d_I, a.K = 1, 1, 100, 4, 64, 8
    a.keys = a.q = a.w = a.idx = 4096
    a.key_row_stride, a.key_batch_stride = 64, 6400
    ok = ctypes.byref(a)
    assert csa._index_ws(ok) > 0
    for field, val, want in [("d_I", 128, csa.CSA_ERR_SHAPE), ("H_I", 9, csa.CSA_ERR_SHAPE),
                             ("K", 0, csa.CSA_ERR_SHAPE), ("key_row_stride", 40, csa.CSA_ERR_SHAPE),
                             ("key_row_stride", 72, csa.CSA_ERR_ALIGNMENT), ("T", 0, csa.CSA_ERR_SHAPE),
                             ("keys", None, csa.CSA_ERR_INVALID_ARG)]:
        b = csa.IndexArgs.from_buffer_copy(a)
        setattr(b, field, val)
        assert csa._index(ctypes.byref(b), None, 0, None) == want, field
    # pool build with an unsupported block length
    b = csa.IndexArgs.from_buffer_copy(a)
    b.pool_out, b.pool_out_len, b.pool_blocks, b.pool_block_len = 4096, 4096, 16, 3
    assert csa._index(ctypes.byref(b), None, 0, None) == csa.CSA_ERR_SHAPE
    # search a pool and build one at once
    b.pool_block_len = 8
    b.pool, b.pool_len, b.pool_cap = 4096, 4096, 128
    assert csa._index(ctypes.byref(b), None, 0, None) == csa.CSA_ERR_UNSUPPORTED
    # workspace missing
    assert csa._index(ok, None, 0, None) == csa.CSA_ERR_WORKSPACE


def test_mx_index_rejects_bad_args_on_host(csa):
    """MXFP4 keys: 32 heads x 128, the exponent plane 4-byte aligned, and the
    code plane 32-byte aligned with 32-byte multiple strides (the packed 4-bit
    copy into the tensor cores' operand layout needs both)."""
    a = csa.IndexArgs()
    a.B, a.n_q, a.T, a.H_I, a.d_I, a.K = 2, 1, 1000, 32, 128, 64
    a.keys = a.q = a.w = a.idx = 4096
    a.key_row_stride, a.key_batch_stride = 64, 64000
    a.key_format = csa.CSA_KEY_MXFP4
    a.key_scales, a.key_scale_row_stride, a.key_scale_batch_stride = 8192, 4, 4000
    ok = ctypes.byref(a)
    assert csa._index_ws(ok) > 0
    assert csa._index(ok, None, 0, None) == csa.CSA_ERR_WORKSPACE      # valid up to the workspace
    for field, val, want in [("keys", 4096 + 16, csa.CSA_ERR_ALIGNMENT),
                             ("key_row_stride", 80, csa.CSA_ERR_ALIGNMENT),
                             ("key_batch_stride", 64016, csa.CSA_ERR_ALIGNMENT),
                             ("key_scale_row_stride", 6, csa.CSA_ERR_ALIGNMENT),
                             ("key_scales", None, csa.CSA_ERR_INVALID_ARG),
                             ("H_I", 8, csa.CSA_ERR_SHAPE), ("d_I", 64, csa.CSA_ERR_SHAPE),
                             ("n_q", 2, csa.CSA_ERR_UNSUPPORTED)]:
        b = csa.IndexArgs.from_buffer_copy(a)
        setattr(b, field, val)
        assert csa._index(ctypes.byref(b), None, 0, None) == want, field


def test_attn_rejects_bad_args_on_host(csa):
    a = csa.AttnArgs()
    a.B, a.n_q, a.H, a.D, a.K, a.n_win = 1, 1, 64, 512, 16, 8
    a.q = a.out = a.kv = a.idx = a.win = 4096
    a.kv_row_stride, a.kv_batch_stride, a.win_row_stride, a.win_batch_stride = 288, 2880, 528, 5280
    a.softmax_scale = 0.044
    for field, val, want in [("H", 24, csa.CSA_ERR_SHAPE), ("D", 448, csa.CSA_ERR_SHAPE),
                             ("kv_row_stride", 272, csa.CSA_ERR_SHAPE),
                             ("kv_row_stride", 296, csa.CSA_ERR_ALIGNMENT),
                             ("win", None, csa.CSA_ERR_INVALID_ARG), ("q", 4100, csa.CSA_ERR_ALIGNMENT),
                             ("n_win", -1, csa.CSA_ERR_SHAPE)]:
        b = csa.AttnArgs.from_buffer_copy(a)
        setattr(b, field, val)
        assert csa._attn(ctypes.byref(b), None, 0, None) == want, field


def test_layer_step_rejects_bad_reuse_source(csa):
    d = (csa.LayerDesc * 1)()
    d[0].mode = csa.CSA_MODE_REUSE
    d[0].reuse_from = 0
    assert csa._layer(d, 1, None, 0, None) == csa.CSA_ERR_INVALID_ARG
    d[0].mode = 7
    assert csa._layer(d, 1, None, 0, None) == csa.CSA_ERR_INVALID_ARG
