"""Pins for the oracle's chained stack and its stand-in glue.

* bf16 rounding: hand-worked ties and steps, and agreement with the bit-level
  round-to-nearest-even of float32 patterns;
* RMSNorm: the closed form of a constant row, unit mean square, scale invariance;
* single-token attention: a hand-made qkv maps each head to its group's v;
* silu: silu(0) = 0, silu(x) - silu(-x) = x, silu(1) = 1 / (1 + e^-1);
* the chain: zero weights leave the residual stream unchanged; a layer whose
  only nonzero weight is `o` adds o . bf16(v) to it.
"""
import math

import numpy as np
import pytest

import oracle.chain as ch


def test_bf16_hand_values():
    one = 1.0
    assert ch.to_bf16(np.array([one]))[0] == 1.0
    assert ch.to_bf16(np.array([1 + 2.0 ** -8]))[0] == 1.0               # tie -> even (down)
    assert ch.to_bf16(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6  # tie -> even (up)
    assert ch.to_bf16(np.array([1 + 2.0 ** -8 + 2.0 ** -20]))[0] == 1 + 2.0 ** -7
    assert ch.to_bf16(np.array([-3.0]))[0] == -3.0
    assert ch.to_bf16(np.array([0.0]))[0] == 0.0


def test_bf16_matches_bit_rounding_of_float32():
    rng = np.random.default_rng(0)
    f = (rng.standard_normal(100000) * np.exp(rng.uniform(-10, 10, 100000))).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16           # RNE on the bit pattern
    want = r.astype(np.uint32).view(np.float32).astype(np.float64)
    assert np.array_equal(ch.to_bf16(f.astype(np.float64)), want)


def test_rmsnorm_constant_row_and_scale():
    h = np.full((1, 64), -0.5)
    eps = 1e-6
    assert np.allclose(ch.rmsnorm(h, eps), -0.5 / math.sqrt(0.25 + eps), rtol=0, atol=1e-15)
    rng = np.random.default_rng(1)
    g = rng.standard_normal((3, 256))
    n = ch.rmsnorm(g, 0.0)
    assert np.allclose(np.mean(n * n, axis=1), 1.0, rtol=1e-12)
    assert np.allclose(ch.rmsnorm(1e3 * g, 0.0), n, rtol=1e-12)


def test_single_token_attention_maps_heads_to_groups():
    d, dkv, hd = 8, 4, 2            # 4 query heads, 2 kv groups of 2 heads
    qkv = np.zeros((1, d + 2 * dkv))
    qkv[0, d + dkv:] = [10, 11, 20, 21]   # v of group 0 = (10, 11), group 1 = (20, 21)
    qkv[0, :d + dkv] = 99.0                # q and k play no part with one token
    out = ch.attention_single_token(qkv, d, dkv, hd)
    assert out.tolist() == [[10, 11, 10, 11, 20, 21, 20, 21]]


def test_silu_identities():
    x = np.linspace(-20, 20, 401)
    assert ch.silu(np.array([0.0]))[0] == 0.0
    assert np.allclose(ch.silu(x) - ch.silu(-x), x, rtol=0, atol=1e-12)
    assert ch.silu(np.array([1.0]))[0] == pytest.approx(1 / (1 + math.exp(-1)), rel=1e-15)


def _zero_layer(d, dkv, f):
    return {"qkv": np.zeros((d + 2 * dkv, d)), "o": np.zeros((d, d)),
            "gate": np.zeros((f, d)), "up": np.zeros((f, d)), "down": np.zeros((d, f))}


def test_chain_zero_weights_is_identity():
    d, dkv, f, hd = 16, 8, 32, 4
    rng = np.random.default_rng(2)
    h = rng.standard_normal((3, d))
    out = ch.chain_forward(h, [_zero_layer(d, dkv, f)] * 3, d, dkv, hd)
    assert np.array_equal(out, h)


def test_chain_attention_only_layer_closed_form():
    # qkv passes the normalized input's first dkv features into v; o adds them
    d, dkv, f, hd = 16, 8, 32, 4
    rng = np.random.default_rng(3)
    h = rng.standard_normal((2, d))
    L = _zero_layer(d, dkv, f)
    L["qkv"][d + dkv + np.arange(dkv), np.arange(dkv)] = 1.0
    L["o"] = rng.standard_normal((d, d))
    out = ch.chain_forward(h, [L], d, dkv, hd)
    xn = ch.to_bf16(h / np.sqrt(np.mean(h * h, axis=1, keepdims=True) + 1e-6))
    v = xn[:, :dkv]
    a = np.concatenate([v[:, (j // 2) * hd:(j // 2 + 1) * hd] for j in range(d // hd)], axis=1)
    assert np.allclose(out, h + a @ L["o"].T, rtol=1e-12, atol=1e-12)


def test_pins_catch_a_dropped_residual():
    d, dkv, f, hd = 16, 8, 32, 4
    h = np.random.default_rng(4).standard_normal((1, d))

    def no_residual(h, layers):
        for L in layers:
            xn = ch.to_bf16(ch.rmsnorm(h))
            h = ch.to_bf16(ch.attention_single_token(xn @ L["qkv"].T, d, dkv, hd)) @ L["o"].T
        return h
    assert not np.array_equal(no_residual(h, [_zero_layer(d, dkv, f)]), h)


def test_bf16_flip_hand_values():
    v = np.array([1.0, 1.0 + 2.0 ** -8 - 2.0 ** -12, 1.0 + 2.0 ** -9, -3.0, -3.0])
    e = np.array([0.0, 2.0 ** -11, 2.0 ** -12, 2.0 ** -7, 2.0 ** -7 + 2.0 ** -10])
    # exact value stays; just below a tie the error reaches it (one bf16 step
    # 2^-7 at 1); mid-interval with a small error nothing moves; -3 -+ 2^-7 are
    # ties that round back to -3 (even); a little further they reach the
    # neighbours -3 -+ 2^-6
    assert ch.bf16_flip(v, e).tolist() == [0.0, 2.0 ** -7, 0.0, 0.0, 2.0 ** -6]


def _rmsnorm_like_the_gpu(h32: np.ndarray, threads: int = 256) -> np.ndarray:
    """fp32 RMSNorm with the reduction structure the bound assumes: each of
    `threads` threads sums every threads-th square sequentially with fp32
    fused multiply-adds, then a tree adds the partial sums."""
    d = h32.shape[1]
    out = np.empty_like(h32)
    for i, row in enumerate(h32):
        part = np.zeros(threads, dtype=np.float32)
        for k in range(0, d, threads):
            blk = row[k:k + threads]
            part[:len(blk)] = (part[:len(blk)].astype(np.float64) + blk.astype(np.float64) ** 2).astype(np.float32)
        while len(part) > 1:
            part = (part[0::2] + part[1::2]).astype(np.float32)
        inv = np.float32(1.0) / np.sqrt(np.float32(part[0] / np.float32(d)) + np.float32(1e-6))
        out[i] = row * inv
    return out.astype(np.float64)


@pytest.mark.parametrize("scale", [1e-3, 1.0, 1e3])
def test_rmsnorm_f32_bound_covers_an_fp32_rmsnorm(scale):
    rng = np.random.default_rng(int(scale * 7) + 1)
    h = (rng.standard_normal((4, 4096)) * scale).astype(np.float32)
    v32 = _rmsnorm_like_the_gpu(h)
    v64 = ch.rmsnorm(h.astype(np.float64))
    err = np.abs(v32 - v64)
    bound = ch.rmsnorm_f32_error(h.astype(np.float64))
    assert np.all(err <= bound)
    # and it is not vacuous: the observed worst case reaches a visible part of it
    assert (err / bound).max() > 0.01


def test_swiglu_f32_bound_covers_fp32_evaluation():
    rng = np.random.default_rng(3)
    g = (rng.standard_normal(100000) * 4).astype(np.float32)
    u = rng.standard_normal(100000).astype(np.float32)
    a32 = (g / (np.float32(1.0) + np.exp(-g)) * u).astype(np.float64)
    g64, u64 = g.astype(np.float64), u.astype(np.float64)
    assert np.all(np.abs(a32 - ch.silu(g64) * u64) <= ch.swiglu_f32_error(g64, u64))
