"""Pins for the oracle's Eq. 1 MinMax int8 quantizer and its fp32 contract.

Independent checks:
* closed forms on rows whose scale is exact (alpha = 1, 1/4) and the
  degenerate constant row;
* invariants fixed by Eq. 1: codes in [0, 255], the row min maps to 0 and the
  row max to 255, codes are monotone in w, and alpha * (q - z) is within
  alpha / 2 of w;
* brute force: q is the integer in [0, 255] nearest to t = w/alpha + z;
* the fp32 contract: float64-then-round equals native IEEE float32 arithmetic
  (numpy float32 scalars) for alpha, z and t.
"""
import numpy as np
import pytest

import oracle
import synth


def test_closed_form_unit_scale():
    w = np.arange(256, dtype=np.float64)[None, :]
    q, a, z = oracle.quantize_minmax(w)
    assert a[0] == 1.0 and z[0] == 0.0
    assert np.array_equal(q[0], np.arange(256))


def test_closed_form_shifted():
    w = np.arange(-128, 128, dtype=np.float64)[None, :]
    q, a, z = oracle.quantize_minmax(w)
    assert a[0] == 1.0 and z[0] == 128.0
    assert np.array_equal(q[0].astype(int), np.arange(256))


def test_closed_form_quarter_scale():
    w = 0.25 * np.arange(256, dtype=np.float64)[None, :] - 3.0
    q, a, z = oracle.quantize_minmax(w)
    assert a[0] == 0.25 and z[0] == 12.0
    assert np.array_equal(q[0].astype(int), np.arange(256))


def test_degenerate_row():
    w = np.full((4, 64), 0.375)
    w[1] = -2.5
    w[2] = 0.0
    w[3] = -2.0 ** -130
    q, a, z = oracle.quantize_minmax(w)
    assert np.all(q == 0)
    # alpha = |min| / 256 (the row's own scale), 2^-126 at the bottom of the range
    assert a.tolist() == [0.375 / 256, 2.5 / 256, 2.0 ** -126, 2.0 ** -126]
    assert z.tolist() == [-256.0, 256.0, 0.0, 2.0 ** -4]
    assert np.array_equal(oracle.dequantize(q, a, z), w)
    for r in (8, 6, 4, 3, 2):
        assert np.array_equal(oracle.dequant_slice(q, a, z, r), w)


@pytest.mark.parametrize("law", ["gauss", "t"])
def test_invariants(law):
    n, k = 64, 512
    bits = (synth.gaussian_weights(n, k, 11) if law == "gauss"
            else synth.student_t_weights(n, k, 12))
    w = synth.f32_from_bf16_bits(bits).astype(np.float64)
    q, a, z = oracle.quantize_minmax(w)
    qi = q.astype(np.int64)
    assert qi.min() >= 0 and qi.max() <= 255
    rows = np.arange(n)
    assert np.all(qi[rows, w.argmin(axis=1)] == 0)
    assert np.all(qi[rows, w.argmax(axis=1)] == 255)
    order = np.argsort(w, axis=1, kind="stable")
    assert np.all(np.diff(np.take_along_axis(qi, order, axis=1), axis=1) >= 0)
    err = np.abs(oracle.dequantize(q, a, z) - w)
    assert np.all(err <= a[:, None].astype(np.float64) * (0.5 + 1e-4))


def test_brute_force_nearest_code():
    w = synth.f32_from_bf16_bits(synth.gaussian_weights(8, 128, 13)).astype(np.float64)
    q, a, z = oracle.quantize_minmax(w)
    cand = np.arange(256, dtype=np.float64)
    for n in range(w.shape[0]):
        a32, z32 = np.float32(a[n]), np.float32(z[n])
        for kk in range(w.shape[1]):
            t = float(np.float32(np.float32(np.float32(w[n, kk]) / a32) + z32))
            d = np.abs(cand - t)
            best = np.flatnonzero(d == d.min())
            # a tie is broken to the even code (round half to even)
            pick = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
            assert q[n, kk] == pick


def test_fp32_contract_matches_native_float32():
    rng = np.random.default_rng(3)
    w32 = (rng.standard_normal((32, 96)) * rng.uniform(1e-3, 10, size=(32, 1))
           + rng.uniform(-1, 1, size=(32, 1))).astype(np.float32)
    q, a, z = oracle.quantize_minmax(w32.astype(np.float64))
    for n in range(w32.shape[0]):
        mn, mx = w32[n].min(), w32[n].max()
        a32 = np.float32(np.float32(mx - mn) / np.float32(255.0))
        z32 = np.float32(-mn / a32)
        assert a[n] == a32 and z[n] == z32
        t32 = (w32[n] / a32 + z32).astype(np.float32)          # float32 ops, elementwise
        q32 = np.clip(np.rint(t32), 0, 255).astype(np.uint8)
        assert np.array_equal(q[n], q32)


def test_fp32_input_rows():
    # the single-layer workload quantizes fp32 weights directly
    w = synth.gaussian_weights(16, 1024, 0, dtype="f32").astype(np.float64)
    q, a, z = oracle.quantize_minmax(w)
    assert q.dtype == np.uint8 and a.dtype == np.float32 and z.dtype == np.float32
    assert np.all(a > 0)


def test_pins_catch_wrong_zero_sign():
    """A planted sign error in z (z = +min/alpha) breaks the row-min -> 0 invariant."""
    w = synth.f32_from_bf16_bits(synth.gaussian_weights(4, 64, 14)).astype(np.float64)
    mn, mx = w.min(axis=1), w.max(axis=1)
    a = (mx - mn) / 255
    bad_z = mn / a
    qbad = np.clip(np.rint(w / a[:, None] + bad_z[:, None]), 0, 255)
    assert not np.all(qbad[np.arange(4), w.argmin(axis=1)] == 0) or \
        not np.all(qbad[np.arange(4), w.argmax(axis=1)] == 255)
