"""MXFP4 indexer keys and their scores (oracle; test infrastructure only).

Format.  DeepSeek-V4.1-Flash architecture database, storage of "decoder
indexer K (m=1)" and "encoder indexer K (m=2)": 128 elements of 4 bits,
"MXFP4 E2M1; E8M0 scales per 32 channels", 4 scale values of 8 bits.  The same
page counts 68 bytes per indexer-K entry (next to 288 for the main KV and 528
for the window).  The indexer that reads these keys has 32 heads of dimension
128 and keeps the top 512 (Model techniques map, "Indexer-selected sparse
attention (DeepSeek Sparse Attention)" row).

Scale rule (a reading: the pages name the format, not the rule).  For each
block of 32 channels, e is the smallest integer with amax <= 6 * 2^e, clamped
to [-127, 127]; amax == 0 gives -127.  This is the window's E8M0 rule with 6,
the largest E2M1 magnitude, in place of 448, so no element is clipped.  Then
    q_i = E2M1_rne_sat(x_i * 2^-e)      (an exact power-of-two scaling)
and the scale byte is e + 127.
Layout of a 128-channel entry: bytes 0..63 hold the codes two per byte, even
channel in the low nibble; bytes 64..67 hold the 4 scale bytes in block order.
Decoded value: val(q_i) * 2^e.

Scores.  S[s] = sum_j w[j] * max(0, <qI[j], k^[s]>), with qI stored as E4M3
codes (the query side keeps the plain E4M3 cast of the current indexer), k^
the decoded MXFP4 key and w fp32.  The dot products are exact.  E4M3 values
are multiples of 2^-9 and E2M1 values multiples of 2^-1.  So, within one
32-channel block, the sum of (q * 2^9) * (code value * 2) is an integer I_b,
and the dot product is sum_b I_b * 2^(e_b - 10).  The blocks are combined
exactly and rounded once to float64.  The weighted head sum is then taken in
float64, heads in ascending order, as for the plain keys.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

from .codecs import e2m1_encode, e2m1_decode, e4m3_int

MX_BLOCK = 32
E2M1_MAX = 6.0


def entry_bytes(dim: int) -> int:
    """Bytes of one MXFP4 entry of `dim` channels: codes, then one scale per block."""
    assert dim % MX_BLOCK == 0
    return dim // 2 + dim // MX_BLOCK


def mx_exponent(amax: np.ndarray) -> np.ndarray:
    """Smallest integer e with amax <= 6 * 2^e, clamped to [-127, 127] (amax == 0 -> -127)."""
    a = np.asarray(amax, dtype=np.float32).astype(np.float64)
    _, f = np.frexp(a)                     # a = m * 2^f, m in [0.5, 1)
    e = f.astype(np.int64) - 1 - 3         # 6 * 2^e < a for this e when a > 0
    for _ in range(4):                     # the answer lies within 3 steps
        bump = a > np.ldexp(E2M1_MAX, e)
        e = e + bump.astype(np.int64)
    e = np.where(a == 0, -127, e)
    return np.clip(e, -127, 127)


def mxfp4_quant_rows(x: np.ndarray) -> np.ndarray:
    """fp32 [N, dim] -> uint8 [N, dim/2 + dim/32]."""
    x = np.asarray(x, dtype=np.float32)
    N, dim = x.shape
    nb = dim // MX_BLOCK
    xb = x.reshape(N, nb, MX_BLOCK)
    e = mx_exponent(np.max(np.abs(xb), axis=2))                       # [N, nb]
    y = xb.astype(np.float64) * np.ldexp(1.0, -e)[:, :, None]          # exact power-of-two scaling
    codes = e2m1_encode(y.astype(np.float32)).reshape(N, dim)          # an fp32 value unless it underflows
                                                                       # below 2^-149, where E2M1 gives +-0 anyway
    out = np.empty((N, entry_bytes(dim)), dtype=np.uint8)
    out[:, :dim // 2] = codes[:, 0::2] | (codes[:, 1::2] << 4)
    out[:, dim // 2:] = (e + 127).astype(np.uint8)
    return out


def _unpack(entries: np.ndarray, dim: int):
    e = np.asarray(entries, dtype=np.uint8)
    N = e.shape[0]
    packed = e[:, :dim // 2]
    codes = np.empty((N, dim), dtype=np.uint8)
    codes[:, 0::2] = packed & 0xF
    codes[:, 1::2] = packed >> 4
    exps = e[:, dim // 2:].astype(np.int64) - 127
    return codes, exps


def mxfp4_dequant_rows(entries: np.ndarray, dim: int = 128) -> np.ndarray:
    """uint8 [N, dim/2 + dim/32] -> float64 [N, dim]."""
    codes, exps = _unpack(entries, dim)
    N = codes.shape[0]
    vals = e2m1_decode(codes).reshape(N, dim // MX_BLOCK, MX_BLOCK)
    return (vals * np.ldexp(1.0, exps)[:, :, None]).reshape(N, dim)


def mx_head_dots(q_codes: np.ndarray, entries: np.ndarray) -> np.ndarray:
    """Exact dot products rounded once to float64: q [H_I, dim] E4M3 codes,
    entries [n, dim/2 + dim/32] MXFP4 keys -> [n, H_I]."""
    q_codes = np.asarray(q_codes)
    H, dim = q_codes.shape
    nb = dim // MX_BLOCK
    assert nb <= 16
    codes, exps = _unpack(entries, dim)                                # [n, dim], [n, nb]
    n = codes.shape[0]
    qi = e4m3_int(q_codes).reshape(H, nb, MX_BLOCK)                    # q * 2^9, |.| <= 229376
    ki = np.rint(e2m1_decode(codes) * 2.0).astype(np.int64).reshape(n, nb, MX_BLOCK)   # value * 2, |.| <= 12
    # I[s, j, b] = sum_i q[j, b, i] * k[s, b, i], |I| < 32 * 229376 * 12 < 2^27
    I = np.einsum("sbi,jbi->sjb", ki, qi)
    e_min = exps.min(axis=1)                                           # [n]
    shift = exps - e_min[:, None]                                      # [n, nb], >= 0
    out = np.empty((n, H), dtype=np.float64)
    # blocks whose exponents lie within 20 of each other: the sum
    # sum_b I_b * 2^(e_b - e_min) is an exact int64 below 2^51 < 2^53, so its
    # float64 conversion is exact and the scaling by 2^(e_min - 10) is too
    narrow = shift.max(axis=1) <= 20
    if narrow.any():
        mult = np.left_shift(np.int64(1), shift[narrow])                # 2^shift
        tot = (I[narrow] * mult[:, None, :]).sum(axis=2)
        out[narrow] = np.ldexp(tot.astype(np.float64), (e_min[narrow] - 10)[:, None])
    # wider spreads: exact rational sum, rounded once
    for s in np.nonzero(~narrow)[0]:
        for j in range(H):
            exact = sum(Fraction(int(I[s, j, b])) * Fraction(2) ** int(exps[s, b] - 10) for b in range(nb))
            out[s, j] = float(exact)
    return out


def mx_index_scores(q_codes: np.ndarray, w: np.ndarray, entries: np.ndarray) -> np.ndarray:
    """float64 [n] scores of n MXFP4 keys for one query (q_codes [H_I, dim], w [H_I])."""
    dots = mx_head_dots(q_codes, entries)
    wj = np.asarray(w, dtype=np.float32).astype(np.float64)
    S = np.zeros(dots.shape[0], dtype=np.float64)
    for j in range(wj.shape[0]):
        S += wj[j] * np.maximum(dots[:, j], 0.0)
    return S
