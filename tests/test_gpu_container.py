"""GPU parity of slice-on-load: the decode GEMV served straight from the int8
container, sliced while streaming by Eq. 6 (clamped) or by the unclamped
Eq. 8 (Extra Precision), against the float64 oracle element by element
within |y - y_ref| <= 1e-3 sum_k |x||W_r| + 1e-6."""
import numpy as np
import pytest
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import synth
from gpu_util import DEV, check_linear, to_dev, weights

pytestmark = pytest.mark.gpu


def gpu_linear_container(x_bits, q, a, z, r, clamp):
    m, k = x_bits.shape
    n = q.shape[0]
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    mq.linear_container(to_dev(x_bits), m, k, to_dev(q), to_dev(a), to_dev(z), n, r, clamp, y)
    mq.device_status()
    return y.cpu().numpy().astype(np.float64)


def _case(law, n, k, seed, r, clamp, m, xseed):
    _, w_vals = weights(law, n, k, seed)
    q, a, z = oracle.quantize_minmax(w_vals)
    x_bits = synth.activations(m, k, xseed)
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    y = gpu_linear_container(x_bits, q, a, z, r, clamp)
    wr = oracle.dequant_slice(q, a, z, r, clamp=clamp)
    return check_linear(y, x_vals, wr, f"container {law} {n}x{k} r={r} clamp={clamp} M={m}")


@pytest.mark.parametrize("clamp", [True, False])
@pytest.mark.parametrize("r", [8, 6, 4, 3, 2])
@pytest.mark.parametrize("m", [1, 4, 16, 32])
def test_container_mistral_up(r, clamp, m):
    _case("t", 14336, 4096, 300, r, clamp, m, 400 + m)


@pytest.mark.parametrize("clamp", [True, False])
@pytest.mark.parametrize("r", [4, 2])
@pytest.mark.parametrize("name,n,k,seed", [
    ("gemma2b_gate", 9216, 2304, 104), ("gemma2b_down", 2304, 9216, 106),
    ("mistral_down", 4096, 14336, 301), ("gemma9b_up", 14336, 3584, 500)])
def test_container_workload_shapes(name, n, k, seed, r, clamp):
    _case("gauss", n, k, seed, r, clamp, 1, 7)


@pytest.mark.parametrize("clamp", [True, False])
@pytest.mark.parametrize("r", [6, 3, 2])
@pytest.mark.parametrize("n,k,m", [(1, 128, 1), (3, 384, 2), (257, 640, 5), (1000, 1152, 9),
                                   (130, 4224, 31)])
def test_container_ragged(n, k, m, r, clamp):
    _case("gauss", n, k, 11 + n, r, clamp, m, 13 + k)


@pytest.mark.parametrize("r", [6, 4, 3, 2])
def test_container_every_byte_and_top_bucket(r):
    # rows holding every container value (and rows all in the top bucket):
    # the extra level 2^r of Eq. 8 and the clamp of Eq. 6 both show up
    n, k = 300, 1024
    rng = np.random.default_rng(r)
    q = rng.integers(0, 256, size=(n, k), dtype=np.uint8)
    q[0] = np.tile(np.arange(256, dtype=np.uint8), 4)
    q[1] = 255
    q[2] = 256 - 2 ** (7 - r)  # lowest value of the extra bucket
    q[3] = 0
    a = (rng.uniform(0.5, 2.0, n) * 1e-3).astype(np.float32)
    z = rng.uniform(0.0, 255.0, n).astype(np.float32)
    for m in (1, 8):
        x_bits = synth.activations(m, k, 50 + m)
        x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
        for clamp in (True, False):
            y = gpu_linear_container(x_bits, q, a, z, r, clamp)
            check_linear(y, x_vals, oracle.dequant_slice(q, a, z, r, clamp=clamp),
                         f"bytes r={r} clamp={clamp} M={m}")
    # the two forms differ exactly on the top-bucket rows
    x_bits = np.full((1, k), 0x3F80, dtype=np.uint16)  # x = 1
    y6 = gpu_linear_container(x_bits, q, a, z, r, True)[0]
    y8 = gpu_linear_container(x_bits, q, a, z, r, False)[0]
    step = a.astype(np.float64) * 2 ** (8 - r)
    assert abs((y8[1] - y6[1]) - k * step[1]) <= 1e-3 * k * step[1]
    assert abs((y8[2] - y6[2]) - k * step[2]) <= 1e-3 * k * step[2]
    assert y8[3] == pytest.approx(y6[3], rel=1e-6, abs=1e-6)


def test_container_matches_planes_within_bound():
    # the container sliced on load and the packed planes serve the same W_r
    n, k, r, m = 4096, 4096, 4, 4
    _, w_vals = weights("t", n, k, 901)
    q, a, z = oracle.quantize_minmax(w_vals)
    x_bits = synth.activations(m, k, 902)
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    yc = gpu_linear_container(x_bits, q, a, z, r, True)
    packed = torch.empty(mq.packed_bytes(n, k, r), dtype=torch.uint8, device=DEV)
    mq.slice_pack(to_dev(q), n, k, r, packed)
    yp = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    mq.linear(to_dev(x_bits), m, k, packed, to_dev(a), to_dev(z), n, r, yp)
    torch.cuda.synchronize()
    wr = oracle.dequant_slice(q, a, z, r)
    tol = oracle.tolerance(x_vals, wr)
    assert np.all(np.abs(yc - yp.cpu().numpy()) <= 2 * tol)


def _prefill_case(law, n, k, seed, r, clamp, m, xseed, rows=None):
    _, w_vals = weights(law, n, k, seed)
    q, a, z = oracle.quantize_minmax(w_vals)
    x_bits = synth.activations(m, k, xseed)
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    y = gpu_linear_container(x_bits, q, a, z, r, clamp)
    label = f"container prefill {law} {n}x{k} r={r} clamp={clamp} M={m}"
    if rows is None:
        return check_linear(y, x_vals, oracle.dequant_slice(q, a, z, r, clamp=clamp), label)
    # rows are quantized independently, so the oracle on a row sample is exact
    return check_linear(y[:, rows], x_vals, oracle.dequant_slice(q[rows], a[rows], z[rows], r, clamp=clamp),
                        label + " (sampled rows)")


@pytest.mark.parametrize("clamp", [True, False])
@pytest.mark.parametrize("r", [8, 6, 4, 3, 2])
@pytest.mark.parametrize("m,n,k", [(33, 300, 1024), (160, 1000, 640), (257, 129, 4224)])
def test_container_prefill_ragged(m, n, k, r, clamp):
    _prefill_case("t", n, k, 31 + n, r, clamp, m, 37 + m)


@pytest.mark.parametrize("clamp", [True, False])
@pytest.mark.parametrize("r", [4, 2])
def test_container_prefill_9b_up_sampled_rows(r, clamp):
    n, k = 14336, 3584
    rng = np.random.default_rng(r)
    rows = np.unique(np.concatenate([rng.choice(n, size=48, replace=False), [0, 127, 128, n - 1]]))
    _prefill_case("gauss", n, k, 500, r, clamp, 2048, 600, rows=rows)


def test_container_prefill_every_byte():
    # every container value in every row, both forms, through the GEMM
    n, k, m = 256, 1024, 64
    rng = np.random.default_rng(3)
    q = np.tile(np.arange(256, dtype=np.uint8), (n, 4))
    for i in range(n):
        rng.shuffle(q[i])
    a = (rng.uniform(0.5, 2.0, n) * 1e-3).astype(np.float32)
    z = rng.uniform(0.0, 255.0, n).astype(np.float32)
    x_bits = synth.activations(m, k, 5)
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    for r in (6, 4, 3, 2):
        for clamp in (True, False):
            y = gpu_linear_container(x_bits, q, a, z, r, clamp)
            check_linear(y, x_vals, oracle.dequant_slice(q, a, z, r, clamp=clamp),
                         f"prefill bytes r={r} clamp={clamp}")
