"""Pins for the oracle's partial RoPE, inverse rotation and bf16 cast (CPU only)."""
import numpy as np
import torch

from oracle import rope, attention, quant


def _cs(angles):
    a = np.asarray(angles, dtype=np.float64)
    return np.stack([np.cos(a), np.sin(a)], axis=1).astype(np.float32)


def test_rotation_hand_values():
    # a quarter turn maps (1, 0) -> (0, 1) and (0, 1) -> (-1, 0) (complex i * z)
    x = np.zeros((2, 512))
    x[0, 448] = 1.0
    x[1, 449] = 1.0
    cs = np.zeros((32, 2), np.float32)
    cs[:, 1] = 1.0                      # cos 0, sin 1
    y = rope.rotate(x, cs)
    assert y[0, 448] == 0.0 and y[0, 449] == 1.0
    assert y[1, 448] == -1.0 and y[1, 449] == 0.0
    # only the last 64 channels move
    z = np.arange(512, dtype=np.float64)[None]
    assert np.array_equal(rope.rotate(z, cs)[0, :448], z[0, :448])


def test_rotation_identity_and_inverse():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5, 512))
    assert np.array_equal(rope.rotate(x, _cs(np.zeros(32))), x)
    cs = _cs(rng.uniform(-50, 50, 32))
    back = rope.rotate(rope.rotate(x, cs), cs, inverse=True)
    # cos^2 + sin^2 of fp32-rounded pairs is 1 within 2^-23
    assert np.allclose(back, x, rtol=0, atol=1e-6)
    # pair norms are kept
    y = rope.rotate(x, cs)
    n0 = x[:, 448::2] ** 2 + x[:, 449::2] ** 2
    n1 = y[:, 448::2] ** 2 + y[:, 449::2] ** 2
    assert np.allclose(n0, n1, rtol=1e-6)


def test_rotation_matches_complex_multiplication():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 512))
    ang = rng.uniform(-3, 3, 32)
    cs = _cs(ang)
    z = x[:, 448::2] + 1j * x[:, 449::2]
    w = z * (cs[:, 0].astype(np.float64) + 1j * cs[:, 1].astype(np.float64))
    y = rope.rotate(x, cs)
    assert np.allclose(y[:, 448::2], w.real, rtol=1e-14, atol=1e-14)
    assert np.allclose(y[:, 449::2], w.imag, rtol=1e-14, atol=1e-14)


def test_relative_position_property():
    # <R(a) q, R(b) k> = <q, R(b - a) k>: the logit sees only the offset
    rng = np.random.default_rng(5)
    q = rng.standard_normal(512)
    k = rng.standard_normal(512)
    a, b = rng.uniform(-2, 2, 32), rng.uniform(-2, 2, 32)
    lhs = rope.rotate(q[None], _cs(a))[0] @ rope.rotate(k[None], _cs(b))[0]
    rhs = q @ rope.rotate(k[None], _cs(b - a))[0]
    assert abs(lhs - rhs) <= 1e-5 * (abs(lhs) + 1)


def test_single_entry_output_is_entry_rotated_back():
    rng = np.random.default_rng(6)
    X = quant.fp4_dequant_rows(quant.fp4_quant_rows(rng.standard_normal((1, 512)).astype(np.float32)))
    q = rng.standard_normal((4, 512)).astype(np.float32)
    cs = _cs(rng.uniform(-3, 3, 32))
    out, lse = rope.attend_rope(q, X, 1 / np.sqrt(512), cs)
    expect = rope.rotate(X, cs, inverse=True)[0]
    assert np.allclose(out, expect[None], rtol=1e-12, atol=1e-12)
    # the nope channels are the entry itself
    assert np.array_equal(out[:, :448], np.broadcast_to(X[0, :448], (4, 448)))


def test_mutation_forward_rotation_on_output_is_caught():
    # rotating the output forward (instead of back) moves a single-entry output
    rng = np.random.default_rng(7)
    X = quant.fp4_dequant_rows(quant.fp4_quant_rows(rng.standard_normal((1, 512)).astype(np.float32)))
    cs = _cs(rng.uniform(0.5, 1.5, 32))
    out, _ = rope.attend_rope(rng.standard_normal((2, 512)).astype(np.float32), X, 0.05, cs)
    wrong = rope.rotate(X, cs)[0]
    assert not np.allclose(out[0, 448:], wrong[448:], atol=1e-3)


def test_query_rotation_changes_logits_like_rotating_keys_back():
    # attending with R(a) q over keys K equals attending with q over R(-a) K
    # (then rotating the output): checks the query is rotated, forward
    rng = np.random.default_rng(8)
    X = rng.standard_normal((40, 512))
    q = rng.standard_normal((3, 512)).astype(np.float32)
    cs = _cs(rng.uniform(-1, 1, 32))
    _, lse = rope.attend_rope(q, X, 0.07, cs)
    _, lse_ref = attention.attend(q, rope.rotate(X, cs, inverse=True), 0.07)
    assert np.allclose(lse, lse_ref, rtol=1e-6)


def test_bf16_round_matches_torch_and_ties():
    rng = np.random.default_rng(9)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    got = rope.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(got, ref)
    # ties go to the even 8-bit significand
    assert rope.bf16_round(np.float32(1 + 2 ** -8)) == 1.0
    assert rope.bf16_round(np.float32(1 + 3 * 2 ** -8)) == 1 + 2 ** -6
    assert rope.bf16_round(np.float32(-(1 + 2 ** -8 + 2 ** -20))) == -(1 + 2 ** -7)


def test_default_angles():
    cs = rope.rope_angles(0)
    assert np.array_equal(cs[:, 0], np.ones(32, np.float32)) and np.array_equal(cs[:, 1], np.zeros(32, np.float32))
    cs = rope.rope_angles(1000)
    assert np.isclose(np.arctan2(cs[0, 1], cs[0, 0]), 1000 - 2 * np.pi * round(1000 / (2 * np.pi)), atol=1e-4)
