"""Cache-entry encodings of the CSA2 step (oracle).

Main-KV entry (a1).  Per the DeepSeek-V4.1 blog ("DeepSeek-V4.1-Flash", CSA2
paragraph: FP4 main KV, "E2M1 format, one E4M3 scale per 16 channels") and the
DeepSeek-V4.1-Flash architecture database (storage of "decoder main KV (m=1)":
512 elements, 256 data bytes + 32 scale bytes of float8_e4m3, 288 B/entry).
For each block of 16 channels, in fp32 arithmetic:
    amax = max |x_i|
    s    = E4M3_rne_sat(amax / 6)            (fp32 division, correctly rounded)
    q_i  = E2M1_rne_sat(x_i / s)             (fp32 division), or +0 for all i if s == 0
Layout: bytes 0..255 hold the 512 codes two per byte, even channel in the low
nibble; bytes 256..287 hold the 32 scale codes in block order.
Decoded value: x^_i = val(q_i) * val(s) (exact: at most 6 significant bits).

Window entry (a2).  Per the architecture database, storage of "SWA window":
FP8 E4M3 with E8M0 scales per 32 channels, 512 data bytes + 16 scale bytes
(528 B); the Training page ("On-policy distillation", Number format) keeps the
sliding-window KV in FP8.  Scale rule (a reading; the pages give none): the
exponent e of each 32-channel block is the smallest integer with
amax <= 448 * 2^e, clamped to [-127, 127] (amax == 0 gives -127), so no element
is clipped; q_i = E4M3_rne_sat(x_i * 2^-e); the scale byte is e + 127.
Decoded value: val(q_i) * 2^e.

Plain E4M3 cast (a2'): indexer keys and queries are stored as E4M3 codes with
no scale.
"""
from __future__ import annotations

import numpy as np

from .codecs import (e2m1_encode, e2m1_decode, e4m3_encode, e4m3_decode, E4M3_MAX)

D = 512
FP4_BLOCK = 16
FP8_BLOCK = 32
FP4_ENTRY_BYTES = D // 2 + D // FP4_BLOCK        # 256 + 32 = 288
FP8_ENTRY_BYTES = D + D // FP8_BLOCK             # 512 + 16 = 528


def fp4_block_scale_codes(x: np.ndarray) -> np.ndarray:
    """[N, 512] fp32 -> [N, 32] E4M3 scale codes (s = E4M3(amax / 6))."""
    xb = np.asarray(x, dtype=np.float32).reshape(x.shape[0], D // FP4_BLOCK, FP4_BLOCK)
    amax = np.max(np.abs(xb), axis=2)
    return e4m3_encode(amax / np.float32(6.0))


def fp4_quant_rows(x: np.ndarray) -> np.ndarray:
    """fp32 (or bf16 values held in fp32) [N, 512] -> uint8 [N, 288]."""
    x = np.asarray(x, dtype=np.float32)
    N = x.shape[0]
    assert x.shape[1] == D
    s_code = fp4_block_scale_codes(x)                              # [N, 32]
    s_val = e4m3_decode(s_code).astype(np.float32)                 # exact in fp32
    xb = x.reshape(N, D // FP4_BLOCK, FP4_BLOCK)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = xb / s_val[:, :, None]                                 # fp32 division
    codes = e2m1_encode(np.where(s_val[:, :, None] == 0, np.float32(0.0), y))
    codes = codes.reshape(N, D)
    out = np.empty((N, FP4_ENTRY_BYTES), dtype=np.uint8)
    out[:, :D // 2] = codes[:, 0::2] | (codes[:, 1::2] << 4)
    out[:, D // 2:] = s_code
    return out


def fp4_dequant_rows(entries: np.ndarray) -> np.ndarray:
    """uint8 [N, 288] -> float64 [N, 512]."""
    e = np.asarray(entries, dtype=np.uint8)
    N = e.shape[0]
    packed = e[:, :D // 2]
    codes = np.empty((N, D), dtype=np.uint8)
    codes[:, 0::2] = packed & 0xF
    codes[:, 1::2] = packed >> 4
    s = e4m3_decode(e[:, D // 2:])                                  # [N, 32]
    return (e2m1_decode(codes).reshape(N, D // FP4_BLOCK, FP4_BLOCK) * s[:, :, None]).reshape(N, D)


def ue8m0_exponent(amax: np.ndarray) -> np.ndarray:
    """Smallest integer e with amax <= 448 * 2^e, clamped to [-127, 127]."""
    a = np.asarray(amax, dtype=np.float32).astype(np.float64)
    _, f = np.frexp(a)                     # a = m * 2^f, m in [0.5, 1)
    e = f.astype(np.int64) - 1 - 9         # below the answer for every a > 0
    for _ in range(4):                     # the answer lies within 3 steps
        bump = a > np.ldexp(E4M3_MAX, e)
        e = e + bump.astype(np.int64)
    e = np.where(a == 0, -127, e)
    return np.clip(e, -127, 127)


def fp8_window_quant_rows(x: np.ndarray) -> np.ndarray:
    """fp32 [N, 512] -> uint8 [N, 528]."""
    x = np.asarray(x, dtype=np.float32)
    N = x.shape[0]
    xb = x.reshape(N, D // FP8_BLOCK, FP8_BLOCK)
    e = ue8m0_exponent(np.max(np.abs(xb), axis=2))                 # [N, 16]
    y = xb.astype(np.float64) * np.ldexp(1.0, -e)[:, :, None]       # exact power-of-two scaling
    codes = e4m3_encode(y.astype(np.float32)).reshape(N, D)        # y is an fp32 value unless it
    out = np.empty((N, FP8_ENTRY_BYTES), dtype=np.uint8)           # underflows below 2^-126,
    out[:, :D] = codes                                             # where E4M3 gives +-0 anyway
    out[:, D:] = (e + 127).astype(np.uint8)
    return out


def fp8_window_dequant_rows(entries: np.ndarray) -> np.ndarray:
    """uint8 [N, 528] -> float64 [N, 512]."""
    e = np.asarray(entries, dtype=np.uint8)
    N = e.shape[0]
    vals = e4m3_decode(e[:, :D]).reshape(N, D // FP8_BLOCK, FP8_BLOCK)
    scale = np.ldexp(1.0, e[:, D:].astype(np.int64) - 127)
    return (vals * scale[:, :, None]).reshape(N, D)


def e4m3_cast(x: np.ndarray) -> np.ndarray:
    """Plain E4M3 codes of fp32 values (indexer keys / queries)."""
    return e4m3_encode(np.asarray(x, dtype=np.float32))
