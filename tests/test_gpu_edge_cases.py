"""GPU parity on the degenerate and adversarial cases of the method, against
closed forms and the float64 oracle (decode GEMV for M <= 32, the tcgen05
GEMM above), within |y - y_ref| <= 1e-3 sum_k |x||W_r| + 1e-6:

* r = 8 on weights that lie on an exact int8 grid: dequantization (Eq. 1)
  then returns the weights themselves, so y = x . W^T in exact arithmetic,
  with nonzero inputs;
* constant rows (max = min): alpha = max(|min| 2^-8, 2^-126), z = -min /
  alpha, every code 0, and W_r = min exactly, so y = min * sum_k x;
* rows whose zero point sits exactly on a code level (the centre code or
  another): most weights dequantize to exactly 0 at every width, so the bound
  shrinks towards 1e-6 while the kernels form y from sums of codes and of x.
"""
import numpy as np
import pytest
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import synth
from gpu_util import DEV, check_linear, gpu_pack, gpu_quantize, to_dev

pytestmark = pytest.mark.gpu

WIDTHS = [8, 6, 4, 3, 2]


def _linear(x_bits, packed, a_d, z_d, n, r, container=None):
    m, k = x_bits.shape
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    if container is None:
        mq.linear(to_dev(x_bits), m, k, packed, a_d, z_d, n, r, y)
    else:
        mq.linear_container(to_dev(x_bits), m, k, container, a_d, z_d, n, r, True, y)
    mq.device_status()
    return y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("m", [1, 4, 32, 33, 96])
def test_r8_exact_int8_grid_nonzero_inputs(m):
    n, k = 192, 4096
    rng = np.random.default_rng(m)
    qg = rng.integers(0, 256, size=(n, k))
    qg[:, 0], qg[:, 1] = 0, 255
    w = (0.5 * (qg - 100.0)).astype(np.float32)      # alpha = 0.5, z = 100 exactly
    q_d, a_d, z_d = gpu_quantize(w, "f32")
    q, a, z = oracle.quantize_minmax(w.astype(np.float64))
    assert np.array_equal(q_d.cpu().numpy(), q) and np.all(a == 0.5) and np.all(z == 100.0)
    assert np.array_equal(oracle.dequant_slice(q, a, z, 8), w.astype(np.float64))
    x_bits = synth.activations(m, k, 900 + m)
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    y = _linear(x_bits, gpu_pack(q_d, 8), a_d, z_d, n, 8)
    # closed form: the product with the original weights
    check_linear(y, x_vals, w.astype(np.float64), f"int8 grid r=8 M={m}")


@pytest.mark.parametrize("r", WIDTHS)
@pytest.mark.parametrize("m", [1, 5, 64])
def test_constant_rows(r, m):
    n, k = 160, 1024
    w = synth.f32_from_bf16_bits(synth.gaussian_weights(n, k, 41)).astype(np.float32)
    consts = [0.0, -0.5, 3.0, 1e-3, -2.0 ** -20, 0.015625]
    for i, c in enumerate(consts):
        w[7 * i + 1, :] = c
    w_bits = synth.bf16_bits_from_f32(w)
    w_vals = synth.f32_from_bf16_bits(w_bits).astype(np.float64)
    q_d, a_d, z_d = gpu_quantize(w_bits, "bf16")
    q, a, z = oracle.quantize_minmax(w_vals)
    assert np.array_equal(q_d.cpu().numpy(), q)
    assert np.array_equal(a_d.cpu().numpy(), a.astype(np.float32))
    assert np.array_equal(z_d.cpu().numpy(), z.astype(np.float32))
    wr = oracle.dequant_slice(q, a, z, r)
    rows = [7 * i + 1 for i in range(len(consts))]
    assert np.array_equal(wr[rows], w_vals[rows])      # min reproduced exactly
    x_bits = synth.activations(m, k, 950 + m)
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    y = _linear(x_bits, gpu_pack(q_d, r), a_d, z_d, n, r)
    check_linear(y, x_vals, wr, f"constant rows r={r} M={m}")
    yc = _linear(x_bits, None, a_d, z_d, n, r, container=q_d)
    check_linear(yc, x_vals, wr, f"constant rows, container, r={r} M={m}")
    # closed form on the constant rows: y = c * sum_k x
    for i in rows:
        cv = w_vals[i, 0]  # the constant after rounding to bf16
        ref = cv * x_vals.sum(axis=1)
        tol = 1e-3 * np.abs(x_vals).sum(axis=1) * abs(cv) + 1e-6
        assert np.all(np.abs(y[:, i] - ref) <= tol)


def _zero_on_code_level(n, k, density, seed, zlevel):
    """Rows with min = -zlevel 2^-7 and max = (255 - zlevel) 2^-7, so alpha =
    2^-7 and z = zlevel exactly, a code level at every width for zlevel = 128
    (the centre) and 64; the rest 0 except a `density` fraction of uniform
    weights inside the range, rounded to bf16."""
    rng = np.random.default_rng(seed)
    lo, hi = -zlevel / 128.0, (255 - zlevel) / 128.0
    w = np.zeros((n, k), dtype=np.float32)
    mask = rng.random((n, k)) < density
    w[mask] = rng.uniform(lo, 0.98 * hi, size=int(mask.sum()))
    cols = rng.integers(0, k, size=(n, 2))
    cols[:, 1] = (cols[:, 0] + 1 + cols[:, 1] % (k - 1)) % k
    w[np.arange(n), cols[:, 0]] = lo
    w[np.arange(n), cols[:, 1]] = hi
    return synth.bf16_bits_from_f32(w)


@pytest.mark.parametrize("r", WIDTHS)
@pytest.mark.parametrize("m", [1, 2, 8, 32, 64])
@pytest.mark.parametrize("k,density,zlevel", [(4096, 0.0, 128), (4096, 0.01, 128), (14336, 0.002, 128),
                                              (4096, 0.0, 64), (14336, 0.002, 64)])
def test_zero_point_on_a_code_level(r, m, k, density, zlevel):
    n = 256
    w_bits = _zero_on_code_level(n, k, density, 17 + k + m, zlevel)
    w_vals = synth.f32_from_bf16_bits(w_bits).astype(np.float64)
    q_d, a_d, z_d = gpu_quantize(w_bits, "bf16")
    q, a, z = oracle.quantize_minmax(w_vals)
    assert np.all(a == 2.0 ** -7) and np.all(z == float(zlevel))
    assert np.array_equal(q_d.cpu().numpy(), q)
    wr = oracle.dequant_slice(q, a, z, r)
    assert (wr == 0.0).mean() > 0.95
    x_bits = synth.activations(m, k, 970 + m)
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    y = _linear(x_bits, gpu_pack(q_d, r), a_d, z_d, n, r)
    ratio = check_linear(y, x_vals, wr, f"z on a code level r={r} M={m} K={k} density={density} z={zlevel}")
    print(f"r={r} M={m} K={k} density={density} z={zlevel}: worst err/tol {ratio:.3f}")
