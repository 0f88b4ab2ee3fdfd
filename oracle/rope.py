"""Partial RoPE around the sparse attention, and the output cast (oracle;
test infrastructure only).

Sources.  DeepSeek-V4.1-Flash architecture database: the global layers use
"partial RoPE (last 64 dims of Q and KV; inverse rotation on attention
output)", with qk_rope_head_dim = 64 of the 512-wide head.  Model techniques
map (DeepSeek-V4.1-Flash), inference kernels: a "Fused RoPE-attention-RoPE-
cast" kernel, and "Post-RoPE KV-cache quantization" (the cache holds latents
whose last 64 channels are already rotated by their own positions).

Reading taken (the pages name the steps, not their formulas):
  1. the last 64 channels of each query head are rotated by the angles of the
     query's position;
  2. the attention runs as in ``attention.attend`` (keys = values = the
     cached, post-RoPE latents);
  3. the last 64 channels of each head's output are rotated back, by the same
     angles negated;
  4. the output is cast to bf16 (round to nearest, ties to even).
Rotation: channel pairs (448 + 2i, 448 + 2i + 1), i = 0..31, treated as the
complex number x + iy and multiplied by e^{i*theta_i}:
    (x, y) -> (x cos - y sin, x sin + y cos)
The angles arrive with the call as fp32 (cos theta_i, sin theta_i) pairs of
the query position (the frequency schedule, YaRN scaling included, is the
caller's: it is not part of the step).  All arithmetic here is float64.
"""
from __future__ import annotations

import numpy as np

from .attention import attend

D = 512
ROPE_DIMS = 64
ROPE_START = D - ROPE_DIMS


def rotate(x: np.ndarray, cs: np.ndarray, inverse: bool = False) -> np.ndarray:
    """Rotate channels [448, 512) of the rows of x ([..., 512]) by the 32 angles
    given as cs [32, 2] = (cos, sin); ``inverse`` rotates by the negated angles.
    Returns a float64 copy (channels below 448 unchanged)."""
    y = np.array(x, dtype=np.float64, copy=True)
    cs = np.asarray(cs, dtype=np.float32).astype(np.float64)
    c, s = cs[:, 0], cs[:, 1]
    if inverse:
        s = -s
    xr = y[..., ROPE_START::2].copy()          # channels 448, 450, ... (real parts)
    xi = y[..., ROPE_START + 1::2].copy()      # channels 449, 451, ... (imaginary parts)
    y[..., ROPE_START::2] = xr * c - xi * s
    y[..., ROPE_START + 1::2] = xr * s + xi * c
    return y


def bf16_round(x) -> np.ndarray:
    """Round fp32 values to bf16 (8 significant bits), nearest, ties to even;
    returned as float64 values.  Written on the fp32 bit pattern: keep the top
    16 bits after adding 0x7FFF plus the lowest kept bit (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def attend_rope(q: np.ndarray, X: np.ndarray, scale: float, cs: np.ndarray, sink=None):
    """Steps 1-3 for one query token: q [H, 512] fp32 values (not yet rotated),
    X [E, 512] dequantised post-RoPE entries, cs [32, 2] the query position's
    angles.  Returns (out [H, 512] float64 before the cast, lse [H])."""
    q_rot = rotate(np.asarray(q, dtype=np.float32).astype(np.float64), cs)
    # attend() takes fp32 query values; the rotated query is rounded to fp32
    # first, as a kernel holding it in fp32 registers would
    out, lse = attend(q_rot.astype(np.float32), X, scale, sink)
    return rotate(out, cs, inverse=True), lse


def rope_angles(position: int, theta: float = 160000.0) -> np.ndarray:
    """Plain RoPE angles of one position as fp32 (cos, sin) pairs [32, 2]:
    theta_i = position * base^(-2i/64).  A convenient default for synthetic
    inputs (base 160,000 is the pages' global-layer rope_theta); the step takes
    any angles."""
    i = np.arange(ROPE_DIMS // 2, dtype=np.float64)
    ang = position * theta ** (-2.0 * i / ROPE_DIMS)
    return np.stack([np.cos(ang), np.sin(ang)], axis=1).astype(np.float32)
