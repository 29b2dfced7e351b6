"""Pins of the Eq. 3 (OmniQuant clipped MinMax) oracle, from what the page and
the arithmetic fix: the reduction to Eq. 1 when gamma = beta = 1, a row worked
out by hand where the clipped scale is exactly 1/64, saturation at both ends,
the half-bucket reconstruction bound inside the clipped range, and the
empty-range rule."""
import numpy as np
import pytest

import oracle
import synth


def test_unit_factors_reduce_to_minmax():
    w = synth.f32_from_bf16_bits(synth.student_t_weights(64, 384, 3)).astype(np.float64)
    ones = np.ones(64)
    q0, a0, z0 = oracle.quantize_minmax(w)
    q1, a1, z1 = oracle.quantize_omniquant(w, ones, ones)
    assert np.array_equal(q0, q1)
    assert np.array_equal(a0.view(np.uint32), a1.view(np.uint32))
    assert np.array_equal(z0.view(np.uint32), z1.view(np.uint32))


def test_hand_worked_row_with_saturation():
    # min = -2, max = 5.96875; beta = gamma = 0.5 clip the range to
    # [-1, 2.984375], whose width 255/64 makes alpha = 1/64 and z = 64 exactly:
    # q = clamp(round_half_even(64 w + 64), 0, 255).
    w = np.array([[-2.0, -1.0, 0.0, 0.5078125, 1.5, 2.984375, 5.96875, -0.0078125]])
    q, a, z = oracle.quantize_omniquant(w, np.array([0.5]), np.array([0.5]))
    assert a[0] == np.float32(1.0 / 64.0)
    assert z[0] == np.float32(64.0)
    #             -2 -> -64 (saturates); -1 -> 0; 0 -> 64; 65/128 -> 96.5 -> 96 (even);
    #             1.5 -> 160; 2.984375 -> 255; 5.96875 -> 446 (saturates); -1/128 -> 63.5 -> 64
    assert q[0].tolist() == [0, 0, 64, 96, 160, 255, 255, 64]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_invariants_inside_and_outside_the_clipped_range(seed):
    rng = np.random.default_rng(seed)
    w = synth.f32_from_bf16_bits(synth.student_t_weights(32, 512, 10 + seed)).astype(np.float64)
    gamma = rng.uniform(0.6, 1.0, 32).astype(np.float32).astype(np.float64)
    beta = rng.uniform(0.6, 1.0, 32).astype(np.float32).astype(np.float64)
    q, a, z = oracle.quantize_omniquant(w, gamma, beta)
    a64, z64 = a.astype(np.float64)[:, None], z.astype(np.float64)[:, None]
    hi = (gamma * w.max(axis=1))[:, None]
    lo = (beta * w.min(axis=1))[:, None]
    assert q.min() >= 0 and q.max() <= 255
    # above the clipped maximum (by more than half a bucket) everything saturates at 255,
    # below the clipped minimum at 0
    assert np.all(q[w > hi + a64] == 255)
    assert np.all(q[w < lo - a64] == 0)
    inside = (w >= lo) & (w <= hi)
    err = np.abs(a64 * (q.astype(np.float64) - z64) - w)
    assert np.all(err[inside] <= (a64 / 2 * (1 + 1e-5) + 1e-12)[np.nonzero(inside)[0]].reshape(-1))


def test_empty_range_rule():
    w = np.array([[0.4, -1.6, 2.5, 3.49]])
    q, a, z = oracle.quantize_omniquant(w, np.array([0.0]), np.array([0.0]))
    # bmin = 0: alpha = 2^-126, z = 0, so every weight saturates by its sign
    assert a[0] == np.float32(2.0 ** -126) and z[0] == 0.0
    assert q[0].tolist() == [255, 0, 255, 255]
    # an all-negative row with gamma = 0 still has a range: gmax = 0, bmin < 0
    wn = np.array([[-1.0, -2.0, -3.0, -0.5]])
    q, a, z = oracle.quantize_omniquant(wn, np.array([0.0]), np.array([0.5]))
    # gmax = 0 * (-0.5) = -0, bmin = 0.5 * -3 = -1.5: range [-1.5, 0] is valid
    assert a[0] == np.float32(1.5 / 255)
    q, a, z = oracle.quantize_omniquant(-wn, np.array([0.0]), np.array([1.0]))
    # all-positive row, gamma = 0: gmax = 0 < bmin = 0.5, inverted
    assert a[0] == np.float32(0.5 / 256) and z[0] == -256.0
    assert q[0].tolist() == [255, 255, 255, 0]   # w / alpha - 256: 0.5 -> 0


def test_pins_catch_an_unclipped_range():
    """A plausible slip, dropping gamma from the range, fails the hand-worked pin."""
    w = np.array([[-2.0, -1.0, 0.0, 0.5078125, 1.5, 2.984375, 5.96875, -0.0078125]])
    q, a, z = oracle.quantize_omniquant(w, np.array([1.0]), np.array([0.5]))
    assert q[0].tolist() != [0, 0, 64, 96, 160, 255, 255, 64]


def test_synthetic_extra_bucket_recipe():
    # the Extra Precision workload: about 2.5% of each row's container values
    # fall in the int2 extra bucket (Eq. 8 code above the Eq. 6 code), as the
    # errata section reports for trained models
    w = synth.f32_from_bf16_bits(synth.extra_bucket_weights(64, 4096, 11)).astype(np.float64)
    q, _, _ = oracle.quantize_minmax(w)
    frac = (oracle.slice_codes(q, 2, clamp=False) != oracle.slice_codes(q, 2)).mean()
    assert 0.02 < frac < 0.035
    # each row's range is pinned, so its extremes map to 0 and 255
    assert (q.min(axis=1) == 0).all() and (q.max(axis=1) == 255).all()
