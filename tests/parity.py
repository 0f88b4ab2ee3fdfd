"""Comparison rules shared by the GPU parity tests.

* Encodings and Top-K of given fp32 scores: bit-exact.
* Indexer Top-K sets: equal, except that every position in the symmetric
  difference must have an oracle score within REL_TIE * |S_K| of the oracle's
  K-th largest score S_K (GPU scores carry fp32 rounding; the oracle's are
  exact), and the GPU row must be ascending with -1 padding.
* Attention outputs: |gpu - oracle| <= ATOL + RTOL * |oracle| per element
  (fp32 outputs; the kernel computes in fp16 operands / fp32 accumulation).
"""
import numpy as np

REL_TIE = 1e-4
RTOL = 2e-3
ATOL = 1e-3


def check_row_format(row: np.ndarray):
    v = row[row >= 0]
    assert np.all(row[len(v):] == -1), "padding must be trailing -1"
    assert np.all(np.diff(v) > 0), "positions must be strictly ascending"


def topk_diff(gpu_row, ora_row, score_of):
    """Return (n_diff, worst relative distance to S_K) and assert the rule."""
    gpu_row = np.asarray(gpu_row)
    ora_row = np.asarray(ora_row)
    check_row_format(gpu_row)
    g = set(gpu_row[gpu_row >= 0].tolist())
    o = set(ora_row[ora_row >= 0].tolist())
    assert len(g) == len(o), (len(g), len(o))
    diff = g ^ o
    if not diff:
        return 0, 0.0
    so = np.array([score_of(p) for p in o])
    S_K = so.min()
    worst = max(abs(score_of(p) - S_K) for p in diff) / max(abs(S_K), 1e-30)
    assert worst <= REL_TIE, f"{len(diff)} differing positions, worst {worst:.3e} relative to S_K"
    return len(diff), worst


def assert_close(gpu, ora, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ora = np.asarray(ora, dtype=np.float64)
    assert gpu.shape == ora.shape, (gpu.shape, ora.shape)
    both_inf = np.isneginf(gpu) & np.isneginf(ora)
    err = np.abs(gpu - ora)
    bound = ATOL + RTOL * np.abs(ora)
    bad = ~((err <= bound) | both_inf)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err - bound, -np.inf)), bad.shape)
        raise AssertionError(f"{what}: {bad.sum()} elements out of tolerance; worst at {i}: "
                             f"gpu={gpu[i]!r} oracle={ora[i]!r}")


def oracle_attend_on(case, cfg, li, t, idx_row, inputs=None):
    """The oracle's attention of layer ``li`` for query ``t`` of ``case``'s
    sequence over the entries of ``idx_row`` (an index row as the GPU wrote
    it, -1 skipped) plus the layer's window rows: used where a near-tie swap
    makes the GPU's Top-K set differ from the oracle's, so that every row's
    attention is still checked against the oracle (on the GPU's own set)."""
    from oracle.attention import attend
    from oracle.quant import fp4_dequant_rows, fp8_window_dequant_rows
    L = cfg.layers[li]
    inp = inputs if inputs is not None else case.inputs(li)
    sel = np.asarray(idx_row)
    sel = sel[sel >= 0].astype(np.int64)
    Xm = fp4_dequant_rows(case.main_entries(L.owner, sel)) if sel.size else np.zeros((0, 512))
    Xw = fp8_window_dequant_rows(inp.window[t:t + cfg.n_win])
    return attend(inp.q[t], np.concatenate([Xm, Xw], axis=0), cfg.softmax_scale, inp.sink)


BF16_HALF_ULP = 2.0 ** -8


def assert_close_bf16(gpu, ora, what=""):
    """bf16 outputs: the fp32 rule plus the bf16 rounding of the result (at most
    half an ulp, 2^-8 relative), since the cast may round either way of a
    result that is itself within the fp32 tolerance."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ora = np.asarray(ora, dtype=np.float64)
    assert gpu.shape == ora.shape, (gpu.shape, ora.shape)
    err = np.abs(gpu - ora)
    bound = ATOL + (RTOL + BF16_HALF_ULP) * np.abs(ora)
    bad = ~(err <= bound)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err - bound, -np.inf)), bad.shape)
        raise AssertionError(f"{what}: {bad.sum()} elements out of tolerance; worst at {i}: "
                             f"gpu={gpu[i]!r} oracle={ora[i]!r}")


BOUNDARY_REL = 1e-5


def check_codes_near_boundaries(gpu_bytes, exact, kind, what=""):
    """Encodings of values that pass through fp32 arithmetic the oracle does in
    float64 (the compressor's exp and division): a GPU code may differ from
    the oracle's only where the exact value lies within BOUNDARY_REL of the
    rounding midpoint between the two codes' values.  kind: "fp4" (288-byte
    entries of 512 channels) or "e4m3" (plain codes).  Returns the number of
    differing codes."""
    from oracle import codecs, quant
    exact = np.asarray(exact, dtype=np.float64)
    gpu_bytes = np.asarray(gpu_bytes, dtype=np.uint8)
    if kind == "e4m3":
        ora = quant.e4m3_cast(exact.astype(np.float32))
        diff = gpu_bytes != ora
        if diff.any():
            mid = (codecs.e4m3_decode(gpu_bytes[diff]) + codecs.e4m3_decode(ora[diff])) / 2
            x = exact[diff]
            assert np.all(np.abs(x - mid) <= BOUNDARY_REL * np.maximum(np.abs(x), 2.0 ** -9)), what
        return int(diff.sum())
    assert kind == "fp4"
    ora = quant.fp4_quant_rows(exact.astype(np.float32))
    n_diff = 0
    for r in range(exact.shape[0]):
        if np.array_equal(gpu_bytes[r], ora[r]):
            continue
        for blk in range(32):
            xs = exact[r, 16 * blk:16 * blk + 16]
            sg, so = gpu_bytes[r, 256 + blk], ora[r, 256 + blk]
            if sg != so:
                # the block scale itself sits at a rounding boundary of amax / 6
                a6 = np.abs(xs).max() / 6
                mid = (codecs.e4m3_decode(np.array([sg])) + codecs.e4m3_decode(np.array([so])))[0] / 2
                assert abs(a6 - mid) <= BOUNDARY_REL * a6, f"{what} row {r} block {blk} scale"
                n_diff += 16
                continue
            s = codecs.e4m3_decode(np.array([sg]))[0]
            for c in range(16):
                b = 8 * blk + c // 2
                cg = (gpu_bytes[r, b] >> (4 * (c % 2))) & 0xF
                co = (ora[r, b] >> (4 * (c % 2))) & 0xF
                if cg != co:
                    mid = (codecs.e2m1_decode(np.array([cg])) + codecs.e2m1_decode(np.array([co])))[0] / 2
                    v = xs[c] / s
                    assert abs(v - mid) <= BOUNDARY_REL * max(abs(v), 0.5), f"{what} row {r} ch {16 * blk + c}"
                    n_diff += 1
    return n_diff
