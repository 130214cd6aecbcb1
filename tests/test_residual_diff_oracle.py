"""Pins of the step-cache decision oracle (CPU only): closed forms, invariances and
a brute-force loop on tiny inputs, chosen so that a dropped absolute value, a
swapped operand or a wrong normaliser fails one of them."""
import math

import numpy as np
import pytest

from oracle.residual_diff import residual_diff, reuse


def test_identical_is_zero_and_reused():
    r = np.random.default_rng(0).standard_normal(1000)
    assert residual_diff(r, r) == 0.0
    assert reuse(r, r, 0.12)


def test_doubling_is_one_and_zero_current_is_one():
    r = np.random.default_rng(1).standard_normal(777)
    assert residual_diff(2 * r, r) == pytest.approx(1.0, abs=1e-15)
    assert residual_diff(np.zeros_like(r), r) == pytest.approx(1.0, abs=1e-15)


def test_normaliser_is_the_previous_residual():
    """Swapping the operands changes the result: |a - b| / |b| is not symmetric."""
    prev = np.array([1.0, -1.0, 2.0, 0.0])
    cur = np.array([1.5, -1.0, 2.0, 1.0])
    assert residual_diff(cur, prev) == pytest.approx(1.5 / 4.0, abs=1e-15)
    assert residual_diff(prev, cur) == pytest.approx(1.5 / 5.5, abs=1e-15)


def test_sign_flip_counts_absolute_values():
    """A dropped absolute value would cancel these differences to zero."""
    prev = np.array([1.0, 1.0, 1.0, 1.0])
    cur = np.array([2.0, 0.0, 2.0, 0.0])
    assert residual_diff(cur, prev) == pytest.approx(1.0, abs=1e-15)


def test_scale_invariance_and_fixed_relative_noise():
    rng = np.random.default_rng(2)
    prev = rng.standard_normal(100_000)
    cur = prev * 1.05                      # every element changes by 5 % of itself
    assert residual_diff(cur, prev) == pytest.approx(0.05, abs=1e-12)
    assert residual_diff(1e-3 * cur, 1e-3 * prev) == pytest.approx(0.05, abs=1e-12)
    assert reuse(cur, prev, 0.12) and not reuse(cur, prev, 0.05 - 1e-9)


def test_zero_previous_residual():
    z = np.zeros(10)
    assert residual_diff(z, z) == 0.0
    assert math.isinf(residual_diff(np.ones(10), z))
    assert not reuse(np.ones(10), z, 1e9)


def test_brute_force_loop_on_tiny_inputs():
    rng = np.random.default_rng(3)
    for n in (1, 2, 3, 17):
        cur, prev = rng.standard_normal(n), rng.standard_normal(n)
        num = den = 0.0
        for a, b in zip(cur.tolist(), prev.tolist()):
            num += abs(a - b)
            den += abs(b)
        assert residual_diff(cur, prev) == pytest.approx(num / den, rel=1e-14)


def test_rejects_mismatched_sizes():
    with pytest.raises(ValueError):
        residual_diff(np.zeros(3), np.zeros(4))
