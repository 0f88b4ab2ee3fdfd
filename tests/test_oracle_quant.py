"""Pins for the oracle's cache-entry encoders (CPU only)."""
import os
from fractions import Fraction

import numpy as np

from oracle import quant, codecs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _examples():
    rows = {}
    with open(os.path.join(GOLDEN, "fp4_block_examples.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, sc, codes, first = line.split()
                rows[name] = (int(sc, 16), [int(ch, 16) for ch in codes], float(first))
    return rows


def _block_row(block):
    x = np.zeros((1, 512), dtype=np.float32)
    x[0, :16] = block
    return x


def check_fp4_examples(quant_rows, dequant_rows):
    ex = _examples()
    blocks = {
        "all_ones": np.ones(16, np.float32),
        "all_zero": np.zeros(16, np.float32),
        "six_block": np.float32([6, 3, -1.5, 0.25] + [0] * 12),
    }
    for name, blk in blocks.items():
        sc, codes, first = ex[name]
        e = quant_rows(_block_row(blk))
        if e.shape != (1, 288) or e[0, 256] != sc:
            return False
        got = [(e[0, i // 2] >> (4 * (i % 2))) & 0xF for i in range(16)]
        if got != codes:
            return False
        if dequant_rows(e)[0, 0] != first:
            return False
    return True


def test_fp4_worked_examples():
    assert check_fp4_examples(quant.fp4_quant_rows, quant.fp4_dequant_rows)


def test_fp4_mutation_swapped_nibbles_is_caught():
    def swapped(x):
        e = quant.fp4_quant_rows(x)
        e[:, :256] = ((e[:, :256] & 0xF) << 4) | (e[:, :256] >> 4)
        return e
    assert not check_fp4_examples(swapped, quant.fp4_dequant_rows)


def test_fp4_mutation_scale_amax_over_4_is_caught():
    def over4(x):
        e = quant.fp4_quant_rows(x)
        xb = x.reshape(x.shape[0], 32, 16)
        e[:, 256:] = codecs.e4m3_encode(np.abs(xb).max(axis=2) / np.float32(4.0))
        return e
    assert not check_fp4_examples(over4, quant.fp4_dequant_rows)


def test_fp4_invariants_random():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((64, 512)) * rng.choice([1e-3, 1, 30, 1e3], size=(64, 1))).astype(np.float32)
    e = quant.fp4_quant_rows(x)
    s = codecs.e4m3_decode(e[:, 256:])                       # [N, 32]
    amax = np.abs(x.reshape(64, 32, 16)).max(axis=2).astype(np.float64)
    # the scale is the nearest E4M3 value to the fp32 quotient amax/6
    q = (amax.astype(np.float32) / np.float32(6.0)).astype(np.float64)
    grid = codecs.e4m3_decode(np.arange(127))
    for i in range(64):
        for b in range(32):
            d = np.abs(grid - q[i, b])
            assert abs(s[i, b] - q[i, b]) == d.min()
    # each element code is the nearest E2M1 value to x/s (unless it saturates at 6);
    # a block whose scale rounds to zero decodes to all zeros
    xh = quant.fp4_dequant_rows(e).reshape(64, 32, 16)
    live = s > 0
    assert np.all(xh[~live] == 0)
    sl = s[live][:, None]
    y = (x.reshape(64, 32, 16)[live] / sl.astype(np.float32)).astype(np.float64)
    v = xh[live] / sl
    mags = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    near = np.abs(np.abs(y)[..., None] - mags).min(axis=-1)
    sat = np.abs(y) > 6
    assert np.all((np.abs(np.abs(v) - np.abs(y)) == near) | (sat & (np.abs(v) == 6)))
    assert np.all(np.sign(v) * np.sign(y) >= 0)


def test_fp4_dequant_exact_in_fp16():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((32, 512)).astype(np.float32)
    xh = quant.fp4_dequant_rows(quant.fp4_quant_rows(x))
    assert np.array_equal(xh.astype(np.float16).astype(np.float64), xh)


def _ceil_log2_exponent(amax):
    """Smallest e with amax <= 448 * 2^e, by exact rational search."""
    a = Fraction(float(amax))
    if a == 0:
        return -127
    e = -200
    while a > Fraction(448) * Fraction(2) ** e:
        e += 1
    return max(-127, min(127, e))


def test_ue8m0_exponent_rule():
    fixed = {448.0: 0, 449.0: 1, 224.0: -1, 224.00002: 0, 0.0: -127, 1.0: -8, 1.75: -8,
             1.7500001: -7, 3e38: 120, 1e-45: -127}
    for a, e in fixed.items():
        assert quant.ue8m0_exponent(np.float32(a)) == e, a
    rng = np.random.default_rng(5)
    a = np.abs(rng.standard_normal(3000) * 10.0 ** rng.integers(-40, 38, 3000)).astype(np.float32)
    a = a[np.isfinite(a)]
    got = quant.ue8m0_exponent(a)
    for ai, gi in zip(a[:600], got[:600]):
        assert gi == _ceil_log2_exponent(ai)


def test_fp8_window_no_clip_and_precision():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((40, 512)) * rng.choice([1e-2, 1, 50], size=(40, 1))).astype(np.float32)
    x[0] = 0
    e = quant.fp8_window_quant_rows(x)
    assert e.shape == (40, 528)
    xh = quant.fp8_window_dequant_rows(e)
    assert np.all(xh[0] == 0) and np.all(e[0, 512:] == 0)      # zero block: e = -127, byte 0
    xb = x.astype(np.float64).reshape(40, 16, 32)
    hb = xh.reshape(40, 16, 32)
    amax = np.abs(xb).max(axis=2)
    # no element is clipped: |x^| <= 448 * 2^e and codes never hit the max unless the value does
    ex = e[:, 512:].astype(np.int64) - 127
    assert np.all(np.abs(hb) <= 448.0 * np.ldexp(1.0, ex)[:, :, None])
    # relative error of normal-range E4M3 is at most 2^-4
    big = np.abs(xb) >= np.ldexp(1.0, ex - 6)[:, :, None]
    err = np.abs(hb - xb)
    assert np.all(err[big] <= np.abs(xb[big]) * 2.0 ** -4)
    assert np.all((amax == 0) | (amax > 448.0 * np.ldexp(1.0, ex - 1)))


def test_plain_cast_is_e4m3():
    x = np.float32([0.1, -3.3, 500.0, 2 ** -12])
    assert np.array_equal(quant.e4m3_cast(x), codecs.e4m3_encode(x))
