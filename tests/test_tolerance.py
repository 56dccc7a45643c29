"""The flip justification of the parity tolerance (tests/helpers.py), on
hand-made BF16 cases: what it admits and what it rejects."""
import numpy as np
import pytest

from helpers import as_f64, rounding_justified


def _bits(vals):
    """Exact BF16 bit patterns of values that BF16 holds."""
    f = np.asarray(vals, np.float32).view(np.uint32)
    assert np.all(f & 0xFFFF == 0)
    return (f >> 16).astype(np.uint16)


ONE, NEXT, NEXT2, PREV = 1.0, 1.0078125, 1.015625, 0.99609375  # BF16 neighbours around 1


def test_storage_values_are_the_neighbours():
    assert list(as_f64(_bits([PREV, ONE, NEXT, NEXT2]))) == [PREV, ONE, NEXT, NEXT2]


def test_rne_value_itself_is_always_admitted():
    exact = np.array([1.001])
    assert rounding_justified(_bits([ONE]), exact, np.array([0.0]))[0]


def test_flip_admitted_only_within_the_bound_of_the_midpoint():
    mid = 0.5 * (ONE + NEXT)
    exact = np.array([mid - 1e-6])                 # RNE(exact) = 1.0, 1e-6 below the midpoint
    assert rounding_justified(_bits([NEXT]), exact, np.array([2e-6]))[0]
    assert not rounding_justified(_bits([NEXT]), exact, np.array([0.5e-6]))[0]


def test_flip_to_the_far_side_is_rejected():
    exact = np.array([0.5 * (ONE + NEXT) - 1e-6])  # closest to 1.0, just below the 1.0|NEXT midpoint
    assert not rounding_justified(_bits([PREV]), exact, np.array([2e-6]))[0]


def test_two_steps_need_a_bound_of_more_than_one_step():
    exact = np.array([1.0001])
    # NEXT2's rounding interval starts at the NEXT|NEXT2 midpoint, 1.01171875
    assert not rounding_justified(_bits([NEXT2]), exact, np.array([0.005]))[0]
    assert rounding_justified(_bits([NEXT2]), exact, np.array([0.0117]))[0]


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_symmetric_in_sign(sign):
    mid = 0.5 * (ONE + NEXT)
    exact = np.array([sign * (mid - 1e-6)])
    assert rounding_justified(_bits([sign * NEXT]), exact, np.array([2e-6]))[0]
    assert not rounding_justified(_bits([-sign * NEXT]), exact, np.array([2e-6]))[0]


def test_zero_and_smallest_values():
    tiny = np.array([np.float32(2.0 ** -133)])     # the smallest BF16 subnormal
    assert rounding_justified(_bits([0.0]), tiny * 0.4, np.array([0.0]))[0]
    assert rounding_justified(_bits(tiny), tiny * 0.6, np.array([0.0]))[0]
    assert not rounding_justified(_bits(tiny), np.array([0.0]), np.array([0.0]))[0]
