"""Each planted mistake in the oracle must be caught by at least one pin.

The oracle source carries compile-time switches (ORC_MUTANT=n) that each plant one
plausible mistake: a wrong code order, a dropped bias, swapped scale/bias, a neighbouring
group, a SiLU sign error, a dropped residual, a dropped sigmoid, ties to the higher index,
no renormalisation, a dropped eps, ties-away rounding, the wrong sub-matrix, and a
normalised layer 0. A mutant that passes every pin would mean the pins cannot see it.
"""
import pytest

import oracle
import oracle_pins as P

MUTANTS = [1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 13, 14]


@pytest.mark.parametrize("m", MUTANTS)
def test_mutant_is_caught(m):
    o = oracle.load(mutant=m)
    assert o.mutant() == m
    caught = []
    for pin in P.ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"mutant {m} passed every pin"
