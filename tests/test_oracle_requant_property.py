"""Property-based pins of the oracle's FP8 requantisation rule, checked in exact
rational arithmetic (``fractions.Fraction``), independently of the oracle's
floating-point search:

* the block exponent n is the smallest integer with max(amax, 1e-4) <= 448 * 2^n;
* every code is the E4M3 value nearest to a / 2^n (ties to the even code), found
  by scanning all finite codes with exact distances;
* no code saturates, because a / 2^n never exceeds 448 in magnitude;
* a block beyond the largest UE8M0 scale (448 * 2^127, past every binary32
  value) is refused rather than given a wrapped scale byte.
"""
import math
from fractions import Fraction

import numpy as np
from hypothesis import assume, given, settings
from hypothesis import strategies as st

from oracle import layer as L
from oracle.formats import decode_e4m3

FINITE = [(c, Fraction(float(decode_e4m3(np.array([c], np.uint8))[0])))
          for c in range(0x7F)]                        # 0x00 .. 0x7E, ascending


def _smallest_n(amax):
    a = max(Fraction(amax), Fraction(1e-4))
    n = -200
    while a > 448 * Fraction(2) ** n:
        n += 1
    return n


def _nearest_code(v):
    """Code of the E4M3 value nearest to the exact rational v; ties to even."""
    a = abs(v)
    best = min(FINITE, key=lambda cm: (abs(cm[1] - a), cm[0] % 2))
    return best[0] | (0x80 if v < 0 else 0)


# With the block scale 2^log_scale (|log_scale| <= 60) these stay within binary32.
floats = st.floats(min_value=-1e20, max_value=1e20, allow_nan=False, allow_infinity=False,
                   allow_subnormal=True)


@settings(max_examples=300, deadline=None)
@given(st.floats(min_value=0.0, max_value=1e30, allow_nan=False, allow_subnormal=True))
def test_block_exponent_is_the_smallest_power_that_fits(amax):
    assert L.ue8m0_exponent_for(amax) == _smallest_n(amax)


@settings(max_examples=40, deadline=None)
@given(st.lists(floats, min_size=128, max_size=128), st.floats(min_value=-60, max_value=60))
def test_requant_codes_are_the_exact_nearest_values(vals, log_scale):
    a = np.array(vals, dtype=np.float64) * 2.0 ** log_scale
    # The activations the layer quantises are binary32 values.
    assume(np.isfinite(a).all() and np.max(np.abs(a)) <= float(np.finfo(np.float32).max))
    codes, sf = L.requant_1x128(a[None, :])
    n = _smallest_n(float(np.max(np.abs(a))))
    assert int(sf[0, 0]) == n + 127
    scale = Fraction(2) ** n
    for v, c in zip(a, codes[0]):
        q = Fraction(float(v)) / scale
        assert abs(q) <= 448
        want = _nearest_code(q)
        # A value that rounds to zero keeps its sign bit; +0 and -0 are both exact.
        if want & 0x7F == 0:
            assert int(c) & 0x7F == 0 and bool(int(c) & 0x80) == (math.copysign(1.0, v) < 0)
        else:
            assert int(c) == want


def test_requant_refuses_blocks_beyond_the_largest_scale():
    import pytest
    ok = np.full((1, 128), 448.0 * 2.0 ** 127)
    _, sf = L.requant_1x128(ok)
    assert int(sf[0, 0]) == 254
    with pytest.raises(ValueError):
        L.requant_1x128(np.nextafter(ok, np.inf))
