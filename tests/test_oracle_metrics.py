"""Pins for the parity checker itself, oracle.metrics.

Every GPU parity assertion goes through it, so a slip here (an abs inside the cosine's
numerator, a maximum over one axis only, a swapped argument, a vacuous branch) would let
every parity test pass. The expected values below are worked out by hand from the
definitions the SageAttention review thread names (reply to reviewer tyTT W1: cosine
similarity, relative L1, RMSE): cos = sum(xy) / sqrt(sum x^2 * sum y^2),
relL1 = sum|x - y| / sum|y|, RMSE = sqrt(mean((x - y)^2)), and max_abs = max|x - y|
over every element.
"""
import math

import numpy as np
import pytest


def test_three_vector_pair_by_hand(oracle_mod):
    # x.y = 2 + 2 + 4 = 8, |x| = |y| = 3 -> cos = 8/9; |x-y| = (1, 1, 0) -> relL1 = 2/5,
    # RMSE = sqrt(2/3), max_abs = 1.
    m = oracle_mod.metrics(np.array([1.0, 2.0, 2.0]), np.array([2.0, 1.0, 2.0]))
    assert m["cos"] == pytest.approx(8.0 / 9.0, abs=1e-15)
    assert m["rel_l1"] == pytest.approx(0.4, abs=1e-15)
    assert m["rmse"] == pytest.approx(math.sqrt(2.0 / 3.0), abs=1e-15)
    assert m["max_abs"] == 1.0


def test_relative_l1_divides_by_the_reference(oracle_mod):
    # x = (3, 0), y = (1, 1): sum|x-y| = 2 + 1 = 3, sum|y| = 2 -> 1.5 (dividing by sum|x|
    # would give 1.0); cos = 3 / (3 * sqrt 2).
    m = oracle_mod.metrics(np.array([3.0, 0.0]), np.array([1.0, 1.0]))
    assert m["rel_l1"] == 1.5
    assert m["cos"] == pytest.approx(1.0 / math.sqrt(2.0), abs=1e-15)
    assert m["rmse"] == pytest.approx(math.sqrt((4.0 + 1.0) / 2.0), abs=1e-15)


def test_identical_and_opposite(oracle_mod):
    y = np.random.default_rng(0).standard_normal((7, 5, 3))
    m = oracle_mod.metrics(y.copy(), y)
    assert m["cos"] == pytest.approx(1.0, abs=1e-15)
    assert m["max_abs"] == 0.0 and m["rel_l1"] == 0.0 and m["rmse"] == 0.0
    m = oracle_mod.metrics(-y, y)
    assert m["cos"] == pytest.approx(-1.0, abs=1e-15)          # an abs in the numerator gives +1
    assert m["max_abs"] == 2.0 * np.abs(y).max()
    assert m["rel_l1"] == pytest.approx(2.0, abs=1e-14)


def test_one_planted_difference_anywhere(oracle_mod):
    # Exactly representable values, so every figure is exact: y is a grid of multiples of
    # 1/4, one element moved by delta = 0.75. max_abs must see it in any position of a
    # 3-D array (a maximum over one axis only misses some positions).
    shape = (4, 6, 8)
    y = (np.arange(np.prod(shape), dtype=np.float64).reshape(shape) % 9 - 4) / 4.0
    n = y.size
    s1 = np.abs(y).sum()
    for idx in [(0, 0, 0), (3, 5, 7), (2, 0, 7), (0, 5, 0)]:
        x = y.copy()
        x[idx] += 0.75
        m = oracle_mod.metrics(x, y)
        assert m["max_abs"] == 0.75, idx
        assert m["rel_l1"] == pytest.approx(0.75 / s1, rel=1e-15)
        assert m["rmse"] == pytest.approx(0.75 / math.sqrt(n), rel=1e-15)
        assert m["cos"] < 1.0


def test_all_zero_output_is_not_similar(oracle_mod):
    # An output of zeros against a nonzero reference is a failure, never cos = 1.
    y = np.array([[0.02, -0.01], [0.03, 0.0]])
    m = oracle_mod.metrics(np.zeros_like(y), y)
    assert m["cos"] == 0.0
    assert m["max_abs"] == 0.03
    assert m["rel_l1"] == pytest.approx(1.0, abs=1e-15)
    # Both zero: identical.
    m = oracle_mod.metrics(np.zeros(3), np.zeros(3))
    assert m["cos"] == 1.0 and m["max_abs"] == 0.0 and m["rel_l1"] == 0.0


def test_shapes_must_agree(oracle_mod):
    # Flattening a transposed output against its reference would compare wrong elements.
    y = np.arange(6.0).reshape(2, 3)
    with pytest.raises(ValueError):
        oracle_mod.metrics(y.T, y)


def test_scale_invariance_of_cos_only(oracle_mod):
    y = np.random.default_rng(1).standard_normal(50)
    m = oracle_mod.metrics(2.0 * y, y)
    assert m["cos"] == pytest.approx(1.0, abs=1e-15)           # cos ignores the scale ...
    assert m["rel_l1"] == pytest.approx(1.0, abs=1e-14)        # ... the other metrics do not
    assert m["max_abs"] == pytest.approx(np.abs(y).max(), rel=1e-15)
