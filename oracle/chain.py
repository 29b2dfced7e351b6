"""A chained decoder stack over the sliced weights (TEST INFRASTRUCTURE).

The Matryoshka Quantization pages quantize the linear layers only; they
define no attention, activation or normalization (section 3.4 on the
explainer page quantizes "the weights of the linear layers", and the
Mix'n'Match paragraph assigns a width per layer). A token's decode step
through a stack of such layers needs some glue between the linears, so this
module fixes a plain stand-in, the reading the CUDA chain follows too:

* pre-norm: RMSNorm without a learned scale, rms(h) = sqrt(mean(h^2) + eps),
  eps = 1e-6, before the qkv and the gate/up projections;
* attention over a context of one token: the softmax over a single score is
  1, so query head j returns the value vector of its key-value group
  j // (n_heads / n_kv_heads) (grouped-query layout q | k | v in qkv);
* SwiGLU MLP: silu(gate) * up, silu(g) = g / (1 + exp(-g));
* residual stream h kept in floating point (float64 here); every linear's
  input is rounded to bfloat16 (round to nearest, ties to even).

Everything is float64; the weights come in dequantized (W_r from
matmul.dequant_slice). No code is shared with the CUDA path.
"""
from __future__ import annotations

import numpy as np


def to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (8 significant bits),
    ties to even, by scaling the significand: v = m 2^e, 0.5 <= |m| < 1."""
    a = np.asarray(a, dtype=np.float64)
    if not np.all(np.isfinite(a)):
        raise ValueError("non-finite value")
    m, e = np.frexp(a)
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def rmsnorm(h: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """h / sqrt(mean(h^2) + eps), per row."""
    h = np.asarray(h, dtype=np.float64)
    return h / np.sqrt(np.mean(h * h, axis=1, keepdims=True) + eps)


def attention_single_token(qkv: np.ndarray, d: int, dkv: int, head_dim: int) -> np.ndarray:
    """Attention output for a context of one token: head j gets v of group
    j // (n_heads / n_kv_heads). qkv columns: q [0, d), k [d, d + dkv),
    v [d + dkv, d + 2 dkv)."""
    n_heads, n_kv = d // head_dim, dkv // head_dim
    per_group = n_heads // n_kv
    v = qkv[:, d + dkv: d + 2 * dkv]
    out = np.empty((qkv.shape[0], d))
    for j in range(n_heads):
        g = j // per_group
        out[:, j * head_dim:(j + 1) * head_dim] = v[:, g * head_dim:(g + 1) * head_dim]
    return out


def silu(g: np.ndarray) -> np.ndarray:
    return g / (1.0 + np.exp(-g))


U32 = 2.0 ** -24  # unit roundoff of fp32 (round to nearest)


def bf16_flip(v: np.ndarray, e: np.ndarray) -> np.ndarray:
    """Largest change of bf16(v') over all v' with |v' - v| <= e: rounding to
    nearest is monotone, so it is reached at v - e or v + e (0 where no
    rounding boundary lies within e of v)."""
    r = to_bf16(v)
    return np.maximum(np.abs(to_bf16(v + e) - r), np.abs(to_bf16(v - e) - r))


def rmsnorm_f32_error(h: np.ndarray, eps: float = 1e-6, threads: int = 256) -> np.ndarray:
    """Bound on |v32 - rmsnorm(h)| for an fp32 RMSNorm of the same fp32 input
    h whose sum of squares is formed by `threads` threads of D / threads
    sequential fused multiply-adds and a reduction tree of depth 16: that sum
    is off by at most (D / threads + 16) u relatively (u = 2^-24); the mean,
    square root, reciprocal and the scaling add 4 u, all relative to |v|."""
    d = h.shape[1]
    gamma = (d / threads + 16) * U32
    return np.abs(rmsnorm(h, eps)) * (gamma / 2 + 4 * U32)


def swiglu_f32_error(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """Bound on |a32 - silu(g) u| for fp32 evaluation of g / (1 + exp(-g)) * u
    on the same fp32 g, u: exp within 2 ulp, the add, the division and the
    product within half an ulp each: 8 u relative."""
    return 8 * U32 * np.abs(silu(g) * u)


def chain_forward(h: np.ndarray, layers, d: int, dkv: int, head_dim: int, eps: float = 1e-6,
                  trace: list | None = None) -> np.ndarray:
    """Runs the layers in order on the residual stream h (M x d).

    layers: list of dicts with float64 weight matrices "qkv" ((d + 2 dkv) x d),
    "o" (d x d), "gate" and "up" (f x d), "down" (d x f). If `trace` is a
    list, the residual stream after each layer is appended to it.
    """
    h = np.asarray(h, dtype=np.float64).copy()
    for L in layers:
        xn = to_bf16(rmsnorm(h, eps))
        qkv = xn @ L["qkv"].T
        a = to_bf16(attention_single_token(qkv, d, dkv, head_dim))
        h1 = h + a @ L["o"].T
        xn1 = to_bf16(rmsnorm(h1, eps))
        act = to_bf16(silu(xn1 @ L["gate"].T) * (xn1 @ L["up"].T))
        h = h1 + act @ L["down"].T
        if trace is not None:
            trace.append(h.copy())
    return h
