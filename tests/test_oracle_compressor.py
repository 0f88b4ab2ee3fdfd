"""Pins for the oracle's m-token compressor (CPU only)."""
import numpy as np

from oracle import compressor as oc


def test_hand_example():
    # gates (0, ln 3): weights 1/4, 3/4
    x = np.array([[[1.0], [3.0]]], np.float32)
    g = np.array([[[0.0], [np.log(3.0)]]], np.float32)
    got = oc.compress(x, g)[0, 0]
    w1 = 1.0 / (1.0 + np.exp(-np.float64(np.float32(np.log(3.0)))))
    assert abs(got - ((1 - w1) * 1.0 + w1 * 3.0)) < 1e-15
    assert abs(got - 2.5) < 1e-6


def test_ratio_one_is_identity():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, 1, 512)).astype(np.float32)
    assert np.array_equal(oc.compress(x, None), x[:, 0].astype(np.float64))


def test_equal_gates_give_the_mean():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 2, 64)).astype(np.float32)
    g = np.repeat(rng.standard_normal((5, 1, 64)).astype(np.float32), 2, axis=1)
    assert np.allclose(oc.compress(x, g), x.astype(np.float64).mean(axis=1), rtol=1e-14, atol=1e-15)


def test_dominant_gate_selects_its_token():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 2, 32)).astype(np.float32)
    g = np.zeros((4, 2, 32), np.float32)
    g[:, 1] = 200.0                                   # exp(-200) ~ 1e-87
    assert np.allclose(oc.compress(x, g), x[:, 1].astype(np.float64), rtol=0, atol=1e-80)


def test_convex_combination_and_token_order_invariance():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((50, 3, 16)).astype(np.float32)
    g = (rng.standard_normal((50, 3, 16)) * 4).astype(np.float32)
    c = oc.compress(x, g)
    lo, hi = x.min(axis=1), x.max(axis=1)
    assert np.all(c >= lo - 1e-12) and np.all(c <= hi + 1e-12)
    perm = [2, 0, 1]
    assert np.allclose(oc.compress(x[:, perm], g[:, perm]), c, rtol=1e-14, atol=1e-15)


def test_mutation_gate_not_normalised_is_caught():
    x = np.ones((1, 2, 4), np.float32)
    g = np.full((1, 2, 4), 1.0, np.float32)
    wrong = (np.exp(g.astype(np.float64)) * x).sum(axis=1)
    assert not np.allclose(wrong, oc.compress(x, g))


def test_group_count():
    assert oc.group_count(0, 2) == 0 and oc.group_count(7, 2) == 3 and oc.group_count(8, 2) == 4
    assert oc.group_count(5, 1) == 5
