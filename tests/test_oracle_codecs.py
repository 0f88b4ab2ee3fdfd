"""Pins for the oracle's scalar codecs (CPU only).

Each codec is checked against something other than itself: a hand-written
golden table, a brute-force nearest-value search, and the ml_dtypes library's
float4_e2m1fn / float8_e4m3fn conversions.  A mutation test plants a wrong
rounding rule into a copy of the oracle and checks that a pin catches it.
"""
import os

import ml_dtypes
import numpy as np
import pytest

from oracle import codecs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _brute_nearest(x, values, codes):
    """Nearest representable by exhaustive search; ties -> even code (lsb 0); saturating."""
    out = []
    vmax = max(abs(v) for v in values if np.isfinite(v))
    for xi in np.asarray(x, dtype=np.float64):
        a = min(abs(xi), vmax)
        best = None
        for v, c in zip(values, codes):
            if not np.isfinite(v) or v < 0 or (v == 0 and c != 0):
                continue
            d = abs(a - v)
            if best is None or d < best[0] or (d == best[0] and (c & 1) == 0 and (best[1] & 1) == 1):
                best = (d, c)
        out.append(best[1])
    return np.array(out)


def test_e2m1_decode_matches_golden_table():
    for code, val in _read("e2m1_table.txt"):
        got = codecs.e2m1_decode(int(code, 16))
        assert got == float(val) and np.signbit(got) == val.startswith("-"), code


def test_e2m1_ties_golden():
    for x, expect in _read("e2m1_ties.txt"):
        c = codecs.e2m1_encode(np.float32(x))
        v = codecs.e2m1_decode(c)
        assert v == float(expect) and np.signbit(v) == expect.startswith("-"), x


def check_e2m1_encode(encode):
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * 3,
        np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 6.5, 7.0, 1e-30, 0.2499999, 0.2500001]),
    ]).astype(np.float32)
    mags = [float(codecs.e2m1_decode(c)) for c in range(8)]
    brute = _brute_nearest(np.abs(x), mags, list(range(8)))
    got = encode(x)
    if not np.array_equal(got & 7, brute):
        return False
    lib = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    return np.array_equal(got, lib)


def test_e2m1_encode_vs_bruteforce_and_ml_dtypes():
    assert check_e2m1_encode(codecs.e2m1_encode)


def test_e2m1_mutation_ties_away_is_caught():
    def ties_away(x):
        x = np.asarray(x, np.float32).astype(np.float64)
        a = np.minimum(np.abs(x), 6.0)
        mags = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
        # nearest, ties away from zero (the wrong rule)
        d = np.abs(a[:, None] - mags[None, :]) - 1e-12 * np.arange(8)[None, :]
        c = np.argmin(d, axis=1)
        return (c | (np.signbit(x) << 3)).astype(np.uint8)
    assert not check_e2m1_encode(ties_away)


def test_e4m3_decode_all_codes_vs_ml_dtypes():
    codes = np.arange(256, dtype=np.uint8)
    ours = codecs.e4m3_decode(codes)
    lib = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], lib[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(lib[~nan]))
    # closed-form facts of the format
    assert np.nanmax(ours) == 448.0 and ours[1] == 2.0 ** -9 and ours[8] == 2.0 ** -6
    assert set(np.nonzero(nan)[0]) == {0x7F, 0xFF}


def check_e4m3_encode(encode):
    rng = np.random.default_rng(12)
    bits = rng.integers(0, 2 ** 32, size=200000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) <= 464.0)]
    x = np.concatenate([x, rng.standard_normal(20000).astype(np.float32),
                        np.float32([0, -0.0, 2 ** -10, -2 ** -10, 3 * 2 ** -11, 448, 464, -464])])
    lib = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    if not np.array_equal(encode(x), lib):
        return False
    # saturation (the library returns NaN beyond the rounding range)
    big = np.float32([465, 1e6, 3e38, -500, -3e38])
    return np.array_equal(encode(big), np.uint8([0x7E, 0x7E, 0x7E, 0xFE, 0xFE]))


def test_e4m3_encode_vs_ml_dtypes_and_saturation():
    assert check_e4m3_encode(codecs.e4m3_encode)


def test_e4m3_encode_vs_bruteforce_midpoints():
    vals = codecs.e4m3_decode(np.arange(127))
    mids = (vals[:-1] + vals[1:]) / 2
    x = np.concatenate([mids, np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
                        np.nextafter(mids.astype(np.float32), np.float32(0))]).astype(np.float32)
    brute = _brute_nearest(x, list(vals), list(range(127)))
    assert np.array_equal(codecs.e4m3_encode(x), brute)


def test_e4m3_mutation_truncation_is_caught():
    def trunc(x):
        x = np.asarray(x, np.float32)
        c = codecs.e4m3_encode(x)
        v = codecs.e4m3_decode(c)
        # round toward zero instead of nearest: step down when we rounded up
        up = np.abs(v) > np.abs(x.astype(np.float64))
        return np.where(up & ((c & 0x7F) > 0), c - 1, c).astype(np.uint8)
    assert not check_e4m3_encode(trunc)


def test_roundtrip_all_codes():
    c4 = np.arange(16, dtype=np.uint8)
    assert np.array_equal(codecs.e2m1_encode(codecs.e2m1_decode(c4).astype(np.float32)), c4)
    c8 = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(codecs.e4m3_encode(codecs.e4m3_decode(c8).astype(np.float32)), c8)


def test_ue8m0_decode():
    b = np.arange(255)
    assert np.array_equal(codecs.ue8m0_decode(b), np.ldexp(1.0, b - 127))
    assert np.isnan(codecs.ue8m0_decode(255))


def test_e4m3_int_exact_multiple():
    c = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(codecs.e4m3_int(c) / 512.0, codecs.e4m3_decode(c))
