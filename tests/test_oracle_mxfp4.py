"""Pins for the oracle's MXFP4 indexer keys and their scores (CPU only)."""
import os
from fractions import Fraction

import numpy as np

from oracle import mxfp4 as mx, indexer, quant, codecs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
DIM = 128


def _examples():
    rows = {}
    with open(os.path.join(GOLDEN, "mxfp4_block_examples.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, sb, codes, first = line.split()
                rows[name] = (int(sb, 16), [int(ch, 16) for ch in codes], float(first))
    return rows


BLOCKS = {
    "all_ones": [1.0] * 32,
    "all_zero": [0.0] * 32,
    "six_block": [6, 3, -1.5, 0.25] + [0] * 28,
    "over_six": [6.5, 5, -0.75] + [0] * 29,
    "small": [0.1, -0.05] + [0] * 30,
}


def check_examples(quant_rows, dequant_rows):
    ex = _examples()
    for name, blk in BLOCKS.items():
        sb, codes, first = ex[name]
        x = np.zeros((1, DIM), dtype=np.float32)
        x[0, :32] = np.float32(blk)
        e = quant_rows(x)
        if e.shape != (1, 68) or e[0, 64] != sb or list(e[0, 65:]) != [0, 0, 0]:
            return False
        got = [(e[0, i // 2] >> (4 * (i % 2))) & 0xF for i in range(4)]
        if got != codes:
            return False
        if dequant_rows(e)[0, 0] != first:
            return False
    return True


def test_worked_examples():
    assert check_examples(mx.mxfp4_quant_rows, mx.mxfp4_dequant_rows)


def test_mutation_floor_scale_rule_is_caught():
    """The OCP-style rule e = floor(log2 amax) - 2 clips 6.5 to 6: the over_six example fails."""
    def floor_rule(x):
        x = np.asarray(x, np.float32)
        N = x.shape[0]
        xb = x.reshape(N, DIM // 32, 32).astype(np.float64)
        amax = np.abs(xb).max(axis=2)
        with np.errstate(divide="ignore"):
            e = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 2, -127).astype(np.int64)
        y = xb * np.ldexp(1.0, -e)[:, :, None]
        codes = codecs.e2m1_encode(y.astype(np.float32)).reshape(N, DIM)
        out = np.empty((N, 68), np.uint8)
        out[:, :64] = codes[:, 0::2] | (codes[:, 1::2] << 4)
        out[:, 64:] = (e + 127).astype(np.uint8)
        return out
    assert not check_examples(floor_rule, mx.mxfp4_dequant_rows)


def test_mutation_swapped_nibbles_is_caught():
    def swapped(x):
        e = mx.mxfp4_quant_rows(x)
        e[:, :64] = ((e[:, :64] & 0xF) << 4) | (e[:, :64] >> 4)
        return e
    assert not check_examples(swapped, mx.mxfp4_dequant_rows)


def test_entry_bytes_match_pages():
    facts = {}
    with open(os.path.join(GOLDEN, "byte_accounting.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, v = line.split()
                facts[k] = int(v)
    assert mx.entry_bytes(DIM) == facts["indexer_k_entry_bytes"] == 68


def _half_spacing(y):
    a = np.abs(y)
    return np.where(a < 2, 0.25, np.where(a < 4, 0.5, 1.0))


def test_invariants_random():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((256, DIM)) * np.exp2(rng.integers(-20, 20, (256, 1)))).astype(np.float32)
    x[3, 32:64] = 0.0                                   # an all-zero block
    e = mx.mxfp4_quant_rows(x)
    exps = e[:, 64:].astype(np.int64) - 127
    xb = x.reshape(256, 4, 32).astype(np.float64)
    amax = np.abs(xb).max(axis=2)
    scale = np.ldexp(1.0, exps)
    # no clipping, and the exponent is the smallest that avoids it
    assert np.all(amax <= 6.0 * scale)
    nz = amax > 0
    assert np.all(amax[nz] > 6.0 * scale[nz] / 2)
    assert np.all(exps[~nz] == -127)
    # every element within half a grid step of its scaled value
    y = xb / scale[:, :, None]
    xh = mx.mxfp4_dequant_rows(e).reshape(256, 4, 32)
    assert np.all(np.abs(xh - xb) <= _half_spacing(y) * scale[:, :, None])
    # decoded values survive a second encode (the bytes may not: a decoded
    # block whose amax fell to 6 * 2^(e-1) or below gets the smaller exponent)
    xh2 = mx.mxfp4_dequant_rows(mx.mxfp4_quant_rows(xh.reshape(256, DIM).astype(np.float32)))
    assert np.array_equal(xh2, xh.reshape(256, DIM))


def _bruteforce_dot(qrow_vals, krow_vals):
    return float(sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(qrow_vals, krow_vals)))


def test_dots_vs_exact_rational_bruteforce():
    rng = np.random.default_rng(5)
    H, n = 3, 24
    q_codes = quant.e4m3_cast(rng.standard_normal((H, DIM)).astype(np.float32))
    k = rng.standard_normal((n, DIM)).astype(np.float32)
    k[0, :32] *= 1e-30                                  # blocks of one key far apart in exponent
    k[0, 96:] *= 1e30
    k[1, 64:96] = 0.0
    entries = mx.mxfp4_quant_rows(k)
    got = mx.mx_head_dots(q_codes, entries)
    qv = codecs.e4m3_decode(q_codes)
    kv = mx.mxfp4_dequant_rows(entries)
    for s in range(n):
        for j in range(H):
            assert got[s, j] == _bruteforce_dot(qv[j], kv[s]), (s, j)


def test_scores_vs_exact_bruteforce_and_head_order():
    rng = np.random.default_rng(6)
    H, n = 4, 16
    q_codes = quant.e4m3_cast(rng.standard_normal((H, DIM)).astype(np.float32))
    w = rng.uniform(0, 1, H).astype(np.float32)
    entries = mx.mxfp4_quant_rows(rng.standard_normal((n, DIM)).astype(np.float32))
    S = mx.mx_index_scores(q_codes, w, entries)
    qv = codecs.e4m3_decode(q_codes)
    kv = mx.mxfp4_dequant_rows(entries)
    for s in range(n):
        ref = 0.0
        for j in range(H):
            ref += float(w[j]) * max(_bruteforce_dot(qv[j], kv[s]), 0.0)
        assert S[s] == ref


def test_mutation_missing_relu_is_caught():
    rng = np.random.default_rng(7)
    H, n = 4, 64
    q_codes = quant.e4m3_cast(rng.standard_normal((H, DIM)).astype(np.float32))
    w = rng.uniform(0, 1, H).astype(np.float32)
    entries = mx.mxfp4_quant_rows(rng.standard_normal((n, DIM)).astype(np.float32))
    dots = mx.mx_head_dots(q_codes, entries)
    no_relu = (dots * w.astype(np.float64)).sum(axis=1)
    assert not np.array_equal(no_relu, mx.mx_index_scores(q_codes, w, entries))


def test_equals_plain_e4m3_keys_when_both_represent_them():
    """Keys on the E2M1 grid with every block's amax exactly 6 are stored
    exactly by both formats (scale 2^0; every E2M1 value is an E4M3 value), so
    the MXFP4 scores equal the plain-key scores of the pinned indexer."""
    rng = np.random.default_rng(8)
    H, n = 8, 200
    grid = np.float32([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    k = grid[rng.integers(0, 8, (n, DIM))] * np.where(rng.random((n, DIM)) < 0.5, -1, 1).astype(np.float32)
    k[:, ::32] = 6.0                                    # amax 6 in every block
    q_codes = quant.e4m3_cast(rng.standard_normal((H, DIM)).astype(np.float32))
    w = rng.uniform(0, 1, H).astype(np.float32)
    entries = mx.mxfp4_quant_rows(k)
    assert np.all(entries[:, 64:] == 127)
    assert np.array_equal(mx.mxfp4_dequant_rows(entries), k.astype(np.float64))
    assert np.array_equal(mx.mx_index_scores(q_codes, w, entries),
                          indexer.index_scores(q_codes, w, quant.e4m3_cast(k)))


def test_stack_with_mxfp4_keys_end_to_end():
    """The oracle's stack run on the pages' indexer shape (32 heads x 128,
    MXFP4 keys, top-512) equals the pieces composed by hand: MXFP4 entries of
    the seeded keys, their scores, the Top-K and the attention over it."""
    from csa_synth import get_config
    from csa_synth import workload as wl
    from oracle.case import SynthCase
    from oracle.attention import attend
    cfg = get_config("decode_mx", B=1, T=3000)
    case = SynthCase(cfg, 0)
    keys = case.keys(0)
    assert keys.shape == (cfg.T, 68)
    assert np.array_equal(keys, mx.mxfp4_quant_rows(wl.index_key(cfg, 0, 0, 0, cfg.T)))
    res = case.run(keep_scores=True)[0]
    inp = case.inputs(0)
    assert inp.qI.shape == (1, 32, 128)
    S = mx.mx_index_scores(inp.qI[0], inp.w[0], keys)
    assert np.array_equal(res.scores[0], S)
    assert np.array_equal(res.idx[0], indexer.topk(S, 512))
    sel = res.idx[0][res.idx[0] >= 0].astype(np.int64)
    X = np.concatenate([quant.fp4_dequant_rows(case.main_entries(0, sel)),
                        quant.fp8_window_dequant_rows(inp.window[0:cfg.n_win])])
    o, l = attend(inp.q[0], X, cfg.softmax_scale, None)
    assert np.array_equal(res.out[0], o) and np.array_equal(res.lse[0], l)
