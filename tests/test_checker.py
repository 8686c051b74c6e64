"""The flip-admissibility rule of the layer check (tests/helpers.py) on
constructed values: a neighbouring code is accepted only when the exact value
sits within the stated window of the decision boundary."""
import numpy as np

import oracle
from helpers import ABS_FLOOR, RHO, _admissible, _quant_h


def test_bf16_tie_admits_both_neighbours():
    lo, hi = 1.0, 1.0 + 2.0 ** -7
    v = (lo + hi) / 2                      # exactly on the rounding boundary
    assert _admissible(v, lo, 0, False, 0.0) and _admissible(v, hi, 0, False, 0.0)


def test_bf16_far_from_boundary_rejects_neighbour():
    v = 1.0 + 2.0 ** -7 * 0.25             # a quarter ulp above 1.0
    assert _admissible(v, 1.0, 0, False, 0.0)
    assert not _admissible(v, 1.0 + 2.0 ** -7, 0, False, 0.0)
    assert not _admissible(v, 1.0 + 2.0 ** -6, 0, False, 0.0)


def test_window_scales_with_row_floor():
    v = 1e-4 + 2.0 ** -21 * 0.3            # tiny value, 0.3 ulp off a bf16 grid point
    near = oracle.bf16_to_double(oracle.bf16_from_double(v))
    other = np.nextafter(np.float32(near), np.float32(1)).item()
    other = oracle.bf16_to_double(oracle.bf16_from_double(near + 2.0 ** -20))
    assert not _admissible(v, other, 0, False, 0.0)           # no floor: rejected
    assert _admissible(v, other, 0, False, 1.0 / RHO * 1e-2)  # a row-scale floor covers it


def test_e4m3_boundary_at_block_exponent():
    e = -3                                   # block scale 2^-3
    # e4m3 neighbours 1.0 and 1.125 (x 2^-3); their tie 1.0625 is itself a bf16 value
    # and rounds to the even code 1.0.  The decision flips between the bf16 values
    # 1.0625 and 1.0703125, so an exact value at their midpoint admits both codes.
    v = 1.06640625 * 2.0 ** e
    a, b = 1.0 * 2.0 ** e, 1.125 * 2.0 ** e
    assert {_quant_h(v * (1 - 1e-6), e, True), _quant_h(v * (1 + 1e-6), e, True)} == {a, b}
    assert _admissible(v, a, e, True, 0.0) and _admissible(v, b, e, True, 0.0)
    assert not _admissible(1.02 * 2.0 ** e, b, e, True, 0.0)
    assert not _admissible(v, 1.25 * 2.0 ** e, e, True, 0.0)
    assert ABS_FLOOR < RHO
