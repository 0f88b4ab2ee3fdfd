"""Scalar number formats, written from their definitions (vectorised NumPy).

Values are handled in float64, which holds every fp32, E4M3 and E2M1 value
exactly; rounding is done explicitly on a power-of-two grid so that no step
depends on a library's float conversion.

E2M1 (OCP Microscaling "FP4"): 1 sign, 2 exponent (bias 1), 1 mantissa bit.
    code c: s = c>>3, e = (c>>1)&3, m = c&1;
    e == 0: value = m * 0.5 (subnormal), else (1 + m/2) * 2^(e-1).
    Magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}; no inf/NaN.
E4M3 (OCP "E4M3FN"): 1 sign, 4 exponent (bias 7), 3 mantissa bits.
    e == 0: value = m * 2^-9; e == 15 and m == 7: NaN; else (1 + m/8) * 2^(e-7).
    Max finite 448; no infinities.
UE8M0: unsigned power of two, value = 2^(byte - 127); 0xFF is NaN.

Encoding (both FP formats): round to nearest, ties to even mantissa, saturate
finite values beyond the largest magnitude to it ("satfinite"); the sign is
kept, so a negative value that rounds to zero gives negative zero.

The main-KV format that uses these is described by the DeepSeek-V4.1 blog,
"DeepSeek-V4.1-Flash" section, CSA2 paragraph ("E2M1 format, one E4M3 scale
per 16 channels"), and by the DeepSeek-V4.1-Flash architecture database, entry
storage facts (main KV FP4 E2M1 + E4M3 per 16; SWA window FP8 E4M3 + E8M0 per
32).
"""
from __future__ import annotations

import numpy as np

E2M1_MAX = 6.0
E4M3_MAX = 448.0


def _as_f64_exact(x) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype != np.float32:
        x = x.astype(np.float32)
    return x.astype(np.float64)


def _round_to_grid(a: np.ndarray, min_exp: int, mant_bits: int, max_val: float) -> np.ndarray:
    """Round |values| ``a`` to the float grid with ``mant_bits`` explicit mantissa
    bits whose smallest normal binade is 2^min_exp (subnormals share that
    binade's spacing); ties to even; saturate at max_val."""
    _, e = np.frexp(a)                 # a = f * 2^e, f in [0.5, 1)  =>  floor(log2 a) = e - 1
    E = np.maximum(e.astype(np.int64) - 1, min_exp)
    spacing = np.ldexp(1.0, E - mant_bits)
    n = np.rint(a / spacing)           # exact quotient; rint = round half to even
    return np.minimum(n * spacing, max_val)


def e2m1_decode(codes) -> np.ndarray:
    c = np.asarray(codes).astype(np.int64) & 0xF
    s = (c >> 3) & 1
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, m * 0.5, (1.0 + m / 2.0) * np.ldexp(1.0, e - 1))
    return np.where(s == 1, -mag, mag)


def e2m1_encode(x) -> np.ndarray:
    """fp32 values -> E2M1 codes (uint8, low nibble)."""
    x = _as_f64_exact(x)
    neg = np.signbit(x)
    v = _round_to_grid(np.abs(x), 0, 1, E2M1_MAX)
    _, e = np.frexp(v)
    E = e.astype(np.int64) - 1
    normal = v >= 1.0
    exp_field = np.where(normal, E + 1, 0)
    mant = np.where(normal, v / np.ldexp(1.0, np.where(normal, E, 0)) * 2.0 - 2.0, v / 0.5)
    code = (exp_field << 1) | mant.astype(np.int64)
    return (code | (neg.astype(np.int64) << 3)).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    c = np.asarray(codes).astype(np.int64) & 0xFF
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 7
    mag = np.where(e == 0, m * np.ldexp(1.0, -9), (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def e4m3_encode(x) -> np.ndarray:
    """fp32 values -> E4M3 codes (uint8), RNE with saturation to +-448."""
    x = _as_f64_exact(x)
    neg = np.signbit(x)
    v = _round_to_grid(np.abs(x), -6, 3, E4M3_MAX)
    _, e = np.frexp(v)
    E = e.astype(np.int64) - 1
    normal = v >= np.ldexp(1.0, -6)
    exp_field = np.where(normal, E + 7, 0)
    scale = np.ldexp(1.0, np.where(normal, E, 0))
    mant = np.where(normal, v / scale * 8.0 - 8.0, v / np.ldexp(1.0, -9))
    code = (exp_field << 3) | mant.astype(np.int64)
    return (code | (neg.astype(np.int64) << 7)).astype(np.uint8)


def ue8m0_decode(b) -> np.ndarray:
    b = np.asarray(b).astype(np.int64)
    return np.where(b == 0xFF, np.nan, np.ldexp(1.0, b - 127))


def e4m3_int(codes) -> np.ndarray:
    """E4M3 values times 2^9 as exact int64 (every finite E4M3 value is a
    multiple of 2^-9, the smallest subnormal)."""
    v = e4m3_decode(codes)
    return np.rint(v * 512.0).astype(np.int64)
