"""Pins for the oracle's dequantize / linear / tolerance / stack.

* exact rational brute force on tiny shapes (fractions.Fraction, Python loops)
  for y[m, n] = sum_k x[m, k] * alpha_n * (S(q[n, k], r) - z_n);
* closed forms: a one-hot x selects a column of W_r; an all-ones x gives
  alpha_n * (2^(8-r) * sum_k code - K * z_n);
* r = 8 on weights that lie exactly on an int8 grid dequantizes exactly;
* the Mix'n'Match stack uses each layer's own width.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

WIDTHS = [8, 6, 4, 3, 2]


def _small(n=3, k=32, m=2, seed=0):
    w = synth.f32_from_bf16_bits(synth.gaussian_weights(n, k, seed)).astype(np.float64)
    x = synth.f32_from_bf16_bits(synth.activations(m, k, seed + 1)).astype(np.float64)
    return w, x


@pytest.mark.parametrize("r", WIDTHS)
def test_exact_rational_brute_force(r):
    w, x = _small()
    q, a, z = oracle.quantize_minmax(w)
    y = oracle.linear(x, oracle.dequant_slice(q, a, z, r))
    s = 8 - r
    for m in range(x.shape[0]):
        for n in range(w.shape[0]):
            acc = Fraction(0)
            for kk in range(w.shape[1]):
                code = oracle.slice_code(int(q[n, kk]), r)
                acc += Fraction(x[m, kk]) * Fraction(float(a[n])) * (code * 2 ** s - Fraction(float(z[n])))
            assert abs(float(acc) - y[m, n]) <= 1e-12 * (1 + abs(float(acc)))


@pytest.mark.parametrize("r", WIDTHS)
def test_one_hot_selects_column(r):
    w, _ = _small(n=5, k=64)
    q, a, z = oracle.quantize_minmax(w)
    wr = oracle.dequant_slice(q, a, z, r)
    for j in [0, 17, 63]:
        x = np.zeros((1, 64))
        x[0, j] = 1.0
        assert np.array_equal(oracle.linear(x, wr)[0], wr[:, j])


@pytest.mark.parametrize("r", WIDTHS)
def test_all_ones_closed_form(r):
    w, _ = _small(n=4, k=128)
    q, a, z = oracle.quantize_minmax(w)
    y = oracle.linear(np.ones((1, 128)), oracle.dequant_slice(q, a, z, r))[0]
    codes = oracle.slice_codes(q, r)
    want = a.astype(np.float64) * (2.0 ** (8 - r) * codes.sum(axis=1) - 128 * z.astype(np.float64))
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12)


def test_int8_grid_round_trips_exactly():
    rng = np.random.default_rng(4)
    qg = rng.integers(0, 256, size=(6, 64))
    qg[:, 0], qg[:, 1] = 0, 255
    w = 0.5 * (qg - 100.0)          # alpha = 0.5, z = 100 exactly
    q, a, z = oracle.quantize_minmax(w)
    assert np.all(a == 0.5) and np.all(z == 100.0)
    assert np.array_equal(oracle.dequant_slice(q, a, z, 8), w)


def test_tolerance_bound_shape_and_floor():
    w, x = _small(n=4, k=64, m=3)
    q, a, z = oracle.quantize_minmax(w)
    wr = oracle.dequant_slice(q, a, z, 4)
    t = oracle.tolerance(x, wr)
    assert t.shape == (3, 4) and np.all(t >= 1e-6)
    assert np.allclose(t, 1e-3 * np.abs(x) @ np.abs(wr).T + 1e-6)


def test_stack_uses_layer_widths():
    widths = [8, 2, 4]
    rng = np.random.default_rng(9)
    lins, lol = [], []
    for layer in range(3):
        for j in range(2):
            lins.append((rng.standard_normal((8, 64)) * 0.02, j))
            lol.append(layer)
    xs = [rng.standard_normal((2, 64)), rng.standard_normal((2, 64))]
    outs = oracle.stack_forward(lins, widths, lol, xs)
    for i, (w, xi) in enumerate(lins):
        q, a, z = oracle.quantize_minmax(w)
        want = oracle.linear(xs[xi], oracle.dequant_slice(q, a, z, widths[lol[i]]))
        assert np.array_equal(outs[i], want)


def test_mixnmatch_widths_pattern():
    wd = synth.mixnmatch_widths(32)
    assert wd[:4] == [8] * 4 and wd[28:] == [8] * 4
    assert wd[4:8] == [4] * 4 and wd[24:28] == [4] * 4
    assert wd[8:24] == [2] * 16
    assert sum(wd) / 32 == 4.0


def test_pins_catch_transposed_matmul():
    w, x = _small(n=3, k=32, m=2)
    q, a, z = oracle.quantize_minmax(w)
    wr = oracle.dequant_slice(q, a, z, 4)
    # x . W (instead of W^T) does not even conform unless shapes collide; use a square case
    sq = np.random.default_rng(2).standard_normal((32, 32))
    xs = np.random.default_rng(3).standard_normal((1, 32))
    assert not np.allclose(oracle.linear(xs, sq), xs @ sq)
    assert oracle.linear(x, wr).shape == (2, 3)


def test_unclamped_dequant_int2_value_set():
    # Eq. 8 (no clamp) at r = 2 over every container value, alpha = 1, z = 0:
    # the errata paragraph's five levels {0, 64, 128, 192, 256}; the top one
    # is reached exactly from q = 224 (= 256 - 2^(s-1)) upward, and below it
    # the two forms agree
    q = np.arange(256, dtype=np.uint8)[None, :]
    one, zero = np.ones(1, np.float32), np.zeros(1, np.float32)
    ep = oracle.dequant_slice(q, one, zero, 2, clamp=False)[0]
    cl = oracle.dequant_slice(q, one, zero, 2)[0]
    assert set(ep.tolist()) == {0.0, 64.0, 128.0, 192.0, 256.0}
    assert np.array_equal(np.nonzero(ep == 256.0)[0], np.arange(224, 256))
    assert np.array_equal(ep[:224], cl[:224]) and np.all(cl[224:] == 192.0)


@pytest.mark.parametrize("r", [6, 4, 3, 2])
def test_unclamped_exact_rational_brute_force(r):
    # y with Eq. 8's unclamped codes, summed in exact rationals; each row's
    # maximum quantizes to q = 255, which lands in the extra bucket 2^r
    w, x = _small(seed=4)
    q, a, z = oracle.quantize_minmax(w)
    assert (q == 255).any(axis=1).all()
    y = oracle.linear(x, oracle.dequant_slice(q, a, z, r, clamp=False))
    s = 8 - r
    for m in range(x.shape[0]):
        for n in range(w.shape[0]):
            acc = Fraction(0)
            for kk in range(w.shape[1]):
                code = (int(q[n, kk]) + 2 ** (s - 1)) >> s  # round half up, no clamp
                acc += Fraction(x[m, kk]) * Fraction(float(a[n])) * (code * 2 ** s - Fraction(float(z[n])))
            assert abs(float(acc) - y[m, n]) <= 1e-12 * (1 + abs(float(acc)))
