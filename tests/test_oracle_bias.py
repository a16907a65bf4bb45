"""Pins for the oracle's bias controller ("MoE router" box, update_bias; teardown
section 6: lower the bias of overloaded experts, raise the others)."""
import numpy as np

import oracle

G = np.float32(1e-3)


def test_equal_load_raises_every_bias():
    b = np.linspace(-0.1, 0.1, 16).astype(np.float32)
    nb = oracle.update_bias(np.full(16, 7, np.int32), b)
    assert np.array_equal(nb, (b + G).astype(np.float32))     # nobody is above the mean


def test_one_overloaded_expert():
    b = np.zeros(4, np.float32)
    nb = oracle.update_bias(np.array([5, 1, 1, 1], np.int32), b)  # mean 2
    assert list(nb) == [-G, G, G, G]


def test_threshold_is_strictly_above_the_mean():
    b = np.zeros(3, np.float32)
    nb = oracle.update_bias(np.array([2, 1, 3], np.int32), b)      # mean 2: 2 is not above
    assert list(nb) == [G, G, -G]
    # a mean that is not an integer: counts [1, 2] -> 1.5
    assert list(oracle.update_bias(np.array([1, 2], np.int32), np.zeros(2, np.float32))) == [G, -G]


def test_step_is_exactly_one_fp32_add():
    rng = np.random.default_rng(0)
    b = rng.uniform(-0.1, 0.1, 256).astype(np.float32)
    c = rng.integers(0, 40, 256).astype(np.int32)
    nb = oracle.update_bias(c, b)
    over = c.astype(np.float32) > np.float32(c.sum()) / np.float32(256)
    assert np.array_equal(nb[over], (b[over] - G).astype(np.float32))
    assert np.array_equal(nb[~over], (b[~over] + G).astype(np.float32))
    # repeated steps drive an always-overloaded expert's bias down linearly
    bb = np.zeros(8, np.float32)
    for _ in range(10):
        bb = oracle.update_bias(np.array([100, 0, 0, 0, 0, 0, 0, 0], np.int32), bb)
    assert abs(float(bb[0]) + 10 * float(G)) < 1e-9 and abs(float(bb[1]) - 10 * float(G)) < 1e-9
