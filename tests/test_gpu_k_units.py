"""GPU parity at K on each width's own unit: every plane row must be a whole
number of 16-byte units, so r = 8 and 4 take any K % 32, r = 6 and 2 any
K % 64, r = 3 any K % 128, and the int8 container any K % 32 at every width.
Such a K ends inside a decode chunk (128 to 512 inputs at M <= 32) and inside
a 64-input stage of the prefill GEMM (M > 32): the bulk copies fill the tail
with zeros, and these tests check that nothing past K reaches y.

Each product is compared element by element with the float64 oracle within
|y - y_ref| <= 1e-3 sum_k |x||W_r| + 1e-6.
"""
import numpy as np
import pytest
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import synth
from gpu_util import DEV, check_linear, gpu_pack, gpu_quantize, to_dev

pytestmark = pytest.mark.gpu

K_UNIT = {8: 32, 4: 32, 6: 64, 2: 64, 3: 128}


def _ks(r):
    u = K_UNIT[r]
    # one unit, a few units, and a long row that ends one unit past a chunk
    return [u, 3 * u, 4096 + u]


CASES = [(r, k) for r in (8, 6, 4, 3, 2) for k in _ks(r)]


@pytest.mark.parametrize("m", [1, 2, 3, 32, 40])
@pytest.mark.parametrize("r,k", CASES)
def test_linear_at_the_width_k_unit(r, k, m):
    n = 200
    w_bits = synth.gaussian_weights(n, k, 500 + k + r)
    w_vals = synth.f32_from_bf16_bits(w_bits).astype(np.float64)
    q_d, a_d, z_d = gpu_quantize(w_bits, "bf16")
    q, a, z = oracle.quantize_minmax(w_vals)
    assert np.array_equal(q_d.cpu().numpy(), q)
    wr = oracle.dequant_slice(q, a, z, r)
    x_bits = synth.activations(m, k, 600 + m + k)
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    packed = gpu_pack(q_d, r)
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    mq.linear(to_dev(x_bits), m, k, packed, a_d, z_d, n, r, y)
    mq.device_status()
    check_linear(y.cpu().numpy().astype(np.float64), x_vals, wr, f"r={r} K={k} M={m}")


@pytest.mark.parametrize("m", [1, 3, 40])
@pytest.mark.parametrize("r", [8, 6, 4, 3, 2])
@pytest.mark.parametrize("k", [32, 96, 4128])
def test_container_at_k_multiple_of_32(r, k, m):
    n = 136
    w_bits = synth.gaussian_weights(n, k, 700 + k + r)
    w_vals = synth.f32_from_bf16_bits(w_bits).astype(np.float64)
    q_d, a_d, z_d = gpu_quantize(w_bits, "bf16")
    q, a, z = oracle.quantize_minmax(w_vals)
    x_bits = synth.activations(m, k, 800 + m + k)
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    mq.linear_container(to_dev(x_bits), m, k, q_d, a_d, z_d, n, r, True, y)
    mq.device_status()
    check_linear(y.cpu().numpy().astype(np.float64), x_vals, oracle.dequant_slice(q, a, z, r),
                 f"container r={r} K={k} M={m}")


def test_stack_with_ragged_k():
    """One Mix'n'Match launch over linears whose K ends off the decode chunk."""
    shapes = [(160, 96, 8), (72, 4160, 2), (300, 4128, 4), (64, 192, 6), (96, 384, 3)]
    lins, widths, refs = [], [], []
    M = 1
    for i, (n, k, r) in enumerate(shapes):
        w_bits = synth.gaussian_weights(n, k, 900 + i)
        w_vals = synth.f32_from_bf16_bits(w_bits).astype(np.float64)
        q_d, a_d, z_d = gpu_quantize(w_bits, "bf16")
        q, a, z = oracle.quantize_minmax(w_vals)
        x_bits = synth.activations(M, k, 950 + i)
        x_d = to_dev(x_bits)
        y = torch.full((M, n), float("nan"), dtype=torch.float32, device=DEV)
        packed = gpu_pack(q_d, r)
        lins.append((x_d, packed, a_d, z_d, y, n, k))
        widths.append(r)
        refs.append((y, synth.f32_from_bf16_bits(x_bits).astype(np.float64), oracle.dequant_slice(q, a, z, r)))
    mq.stack_forward(lins, list(range(len(lins))), widths, M)
    mq.device_status()
    for (y, xv, wr), (n, k, r) in zip(refs, shapes):
        check_linear(y.cpu().numpy().astype(np.float64), xv, wr, f"batched r={r} N={n} K={k}")
