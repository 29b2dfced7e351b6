"""Pins for the oracle's slicing operator (Eq. 6 / Eq. 8).

What fixes the operator, independently of the oracle's own code:
* the pages' worked values (tests/golden/slicing_worked_examples.txt);
* the pages' int2 value sets with and without the clamp (golden file);
* S(q, c) = q, range and multiple-of-2^(c-r) properties (Eq. 6 itself);
* brute force: S(q, r) is the representable value nearest to q, ties upward
  (the "first dropped bit decides" rule of the same paragraph);
* the bucket boundaries implied by round-half-up and the clamp.
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
WIDTHS = [8, 6, 4, 3, 2]


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def test_worked_examples_from_pages():
    rows = _rows("slicing_worked_examples.txt")
    assert rows, "golden file empty"
    for q, r, v in rows:
        assert oracle.slice_value(int(q), int(r)) == int(v)


def test_int2_value_sets_with_and_without_clamp():
    for eq, r, *vals in _rows("slicing_value_sets.txt"):
        got = {oracle.slice_value(q, int(r), clamp=(eq == "eq6")) for q in range(256)}
        assert got == {int(v) for v in vals}, eq


@pytest.mark.parametrize("r", WIDTHS)
def test_range_and_multiples(r):
    s = 8 - r
    for q in range(256):
        code = oracle.slice_code(q, r)
        assert 0 <= code <= (1 << r) - 1
        assert oracle.slice_value(q, r) % (1 << s) == 0


def test_full_width_is_identity():
    assert all(oracle.slice_value(q, 8) == q for q in range(256))
    assert np.array_equal(oracle.slice_table(8), np.arange(256))


@pytest.mark.parametrize("r", WIDTHS)
def test_brute_force_nearest_representable_ties_up(r):
    s = 8 - r
    reps = [k << s for k in range(1 << r)]
    for q in range(256):
        best = min(reps, key=lambda v: (abs(q - v), -v))  # nearest; on a tie the larger
        assert oracle.slice_value(q, r) == best, (q, r)


def test_bucket_boundaries_r2():
    # round half up on q/64 then clamp: 0-31 -> 0, 32-95 -> 64, 96-159 -> 128, 160-255 -> 192
    expect = [0] * 32 + [64] * 64 + [128] * 64 + [192] * 96
    assert [oracle.slice_value(q, 2) for q in range(256)] == expect


def test_half_point_rounds_up():
    # q/2^(8-r) exactly x.5: the dropped MSB is 1, so the value rounds up
    assert oracle.slice_code(32, 2) == 1      # 0.5 -> 1
    assert oracle.slice_code(96, 2) == 2      # 1.5 -> 2 (not to even)
    assert oracle.slice_code(8, 4) == 1       # 0.5 -> 1
    assert oracle.slice_code(1, 7) == 1       # 0.5 -> 1


def test_unclamped_top_bucket():
    # Eq. 8 reaches 2^r only from the top of the range
    for r in [2, 3, 4, 6]:
        s = 8 - r
        top = [q for q in range(256) if oracle.slice_code(q, r, clamp=False) == (1 << r)]
        assert top == list(range(256 - (1 << (s - 1)), 256))


def test_vectorized_codes_match_scalar():
    q = np.random.default_rng(5).integers(0, 256, size=(7, 64))
    for r in WIDTHS:
        want = np.vectorize(lambda v: oracle.slice_code(int(v), r))(q)
        assert np.array_equal(oracle.slice_codes(q, r), want)


def test_pins_catch_floor_rounding():
    """A planted mistake (floor instead of round-half-up) fails the page's 53 -> 64 pin."""
    def floor_slice(q, r):
        s = 8 - r
        return min(q >> s, (1 << r) - 1) << s
    assert floor_slice(53, 2) != 64


def test_pins_catch_missing_clamp():
    def noclamp(q, r):
        s = 8 - r
        return ((q + (1 << (s - 1))) >> s) << s
    assert noclamp(234, 2) != 192
