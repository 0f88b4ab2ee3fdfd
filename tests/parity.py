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
