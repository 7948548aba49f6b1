"""The block-scaled parity checker itself (tests/mx_parity.py), on the CPU.

hidden_check accepts a GPU hidden value that differs from the oracle's only
where the oracle marks the element as near a rounding boundary, and only by
one E4M3 step; these cases pin both halves of that rule, so a checker that let
a scale or code error through would fail here.
"""
from __future__ import annotations

import numpy as np
import pytest

import mx_parity as MX
import oracle.oracle as O


def _row(values, amax=400.0):
    """A block of 32 whose maximum sets scale 2^0 (400: away from the scale
    boundaries at 224 and 448) and whose first entries are `values`."""
    h = np.zeros((1, 32))
    h[0, -1] = amax
    h[0, : len(values)] = values
    return h


def test_identical_values_pass_without_flips():
    rng = np.random.default_rng(0)
    h = rng.normal(0, 1, (3, 128)) * rng.normal(0, 1, (3, 128))
    v = O.mx_dequantize(*O.mx_quantize(h))
    assert MX.hidden_check(h, v)["flips"] == 0


def test_one_step_at_an_exact_midpoint_is_allowed():
    # 1.0625 lies halfway between the E4M3 values 1.0 and 1.125 (scale 2^0):
    # round-to-nearest-even gives 1.0, a sum a hair larger gives 1.125.
    h = _row([1.0625])
    v = O.mx_dequantize(*O.mx_quantize(h))
    assert v[0, 0] == 1.0
    v[0, 0] = 1.125
    r = MX.hidden_check(h, v)
    assert r["flips"] == 1 and r["dv"][0, 0] == pytest.approx(0.125)


def test_one_step_away_from_a_boundary_fails():
    h = _row([1.03])                  # nearest 1.0, far from the 1.0625 midpoint
    v = O.mx_dequantize(*O.mx_quantize(h))
    v[0, 0] = 1.125
    with pytest.raises(AssertionError):
        MX.hidden_check(h, v)


def test_two_steps_at_a_midpoint_fail():
    h = _row([1.0625])
    v = O.mx_dequantize(*O.mx_quantize(h))
    v[0, 0] = 1.25
    with pytest.raises(AssertionError):
        MX.hidden_check(h, v)


def test_a_block_off_by_a_factor_of_two_fails():
    rng = np.random.default_rng(1)
    h = rng.normal(0, 1, (2, 64))
    v = O.mx_dequantize(*O.mx_quantize(h))
    v[1, 32:] *= 2.0                  # the scale of one block read from elsewhere
    with pytest.raises(AssertionError):
        MX.hidden_check(h, v)


def test_block_maximum_on_a_scale_boundary_allows_the_other_scale():
    # amax exactly 448 * 2^0: a larger sum would take scale 2^1, whose grid is
    # twice as coarse; the other elements may then sit one coarse step away.
    h = _row([3.3], amax=448.0)
    v = O.mx_dequantize(*O.mx_quantize(h))
    v[0, 0] = 3.5                     # 3.3 at scale 2^1: 1.65 -> 1.625 -> 3.25 or 3.5
    assert MX.hidden_check(h, v)["flips"] == 1
