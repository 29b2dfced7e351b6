"""GPU parity of the fused unpack -> dequantize -> matmul (decode GEMV,
M <= 32) against the float64 oracle, element by element within
|y - y_ref| <= 1e-3 sum_k |x||W_r| + 1e-6."""
import numpy as np
import pytest
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import synth
from gpu_util import DEV, check_linear, gpu_linear, gpu_pack, to_dev, weights

pytestmark = pytest.mark.gpu

WIDTHS = [8, 6, 4, 3, 2]


def _case(law, n, k, seed, r, m, xseed, dtype="bf16"):
    w_host, w_vals = weights(law, n, k, seed, dtype)
    q, a, z = oracle.quantize_minmax(w_vals)
    packed = gpu_pack(to_dev(q), r)
    x_bits = synth.activations(m, k, xseed)
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    y = gpu_linear(x_bits, packed, to_dev(a), to_dev(z), n, r)
    return check_linear(y, x_vals, oracle.dequant_slice(q, a, z, r), f"{law} {n}x{k} r={r} M={m}")


@pytest.mark.parametrize("r", [8, 4, 2])
def test_single_linear_fp32_weights(r):
    _case("gauss", 512, 1024, 0, r, 1, 1, dtype="f32")


@pytest.mark.parametrize("m", [1, 4, 8])
@pytest.mark.parametrize("name,n,k,seed", [
    ("q", 2304, 2304, 100), ("gate", 9216, 2304, 104), ("down", 2304, 9216, 106)])
def test_gemma2b_layer_r4(name, n, k, seed, m):
    _case("gauss", n, k, seed, 4, m, 200 + m)


@pytest.mark.parametrize("r", [2, 4, 8])
@pytest.mark.parametrize("m", [1, 4, 16, 32])
@pytest.mark.parametrize("name,n,k,seed", [("up", 14336, 4096, 300), ("down", 4096, 14336, 301)])
def test_mistral_mlp_heavy_tail(name, n, k, seed, r, m):
    _case("t", n, k, seed, r, m, 400 + m)


@pytest.mark.parametrize("r", WIDTHS)
@pytest.mark.parametrize("m", [1, 2, 3, 7, 8, 9, 15, 17, 24, 31, 32])
def test_all_widths_all_batch_sizes(r, m):
    _case("gauss", 300, 1152, 11 + r, r, m, 50 + m)


@pytest.mark.parametrize("r", WIDTHS)
@pytest.mark.parametrize("n,k", [(1, 128), (5, 128), (127, 256), (129, 384), (1000, 896), (257, 2176)])
def test_ragged_shapes(r, n, k):
    _case("t", n, k, n + k, r, 3, n)


@pytest.mark.parametrize("r", WIDTHS)
def test_one_hot_selects_dequantized_column(r):
    n, k = 256, 512
    w_host, w_vals = weights("gauss", n, k, 77, "bf16")
    q, a, z = oracle.quantize_minmax(w_vals)
    packed = gpu_pack(to_dev(q), r)
    wr = oracle.dequant_slice(q, a, z, r)
    for j in [0, 1, 255, 511]:
        x = np.zeros((1, k), dtype=np.float32)
        x[0, j] = 1.0
        xb = synth.bf16_bits_from_f32(x)
        y = gpu_linear(xb, packed, to_dev(a), to_dev(z), n, r)[0]
        assert np.allclose(y, wr[:, j], rtol=1e-6, atol=1e-6 * np.abs(wr).max())


@pytest.mark.parametrize("r", WIDTHS)
def test_int8_grid_exact_and_zero_input(r):
    n, k = 64, 256
    rng = np.random.default_rng(r)
    qg = rng.integers(0, 256, size=(n, k))
    qg[:, 0], qg[:, 1] = 0, 255
    w = (0.5 * (qg - 100.0)).astype(np.float32)
    q, a, z = oracle.quantize_minmax(w.astype(np.float64))
    packed = gpu_pack(to_dev(q), r)
    xz = np.zeros((2, k), np.uint16)
    y = gpu_linear(xz, packed, to_dev(a), to_dev(z), n, r)
    assert np.all(y == 0.0)


def test_outputs_fully_overwritten():
    """y is NaN-filled before the call; every element must be written."""
    _case("gauss", 777, 640, 5, 4, 5, 6)


def test_timeout_path_reports_and_recovers():
    """A wait limit of 0 makes every pipeline wait give up at once: the kernel
    must set the error flag, drain its copies and exit; the next normal call
    must succeed."""
    n, k, r = 512, 1024, 4
    w_host, w_vals = weights("gauss", n, k, 1, "bf16")
    q, a, z = oracle.quantize_minmax(w_vals)
    packed = gpu_pack(to_dev(q), r)
    x_bits = synth.activations(1, k, 2)
    x_d = to_dev(x_bits)
    y = torch.zeros((1, n), dtype=torch.float32, device=DEV)
    mq.debug_set_wait_limit_ns(0)
    try:
        mq.linear(x_d, 1, k, packed, to_dev(a), to_dev(z), n, r, y)
        with pytest.raises(mq.MQError) as e:
            mq.device_status()
        assert e.value.status == mq.MQ_ERR_TIMEOUT
    finally:
        mq.debug_set_wait_limit_ns(2_000_000_000)
    mq.device_status()  # flag cleared
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    y2 = gpu_linear(x_bits, packed, to_dev(a), to_dev(z), n, r)
    check_linear(y2, x_vals, oracle.dequant_slice(q, a, z, r), "after timeout")


def test_repeat_calls_consistent():
    n, k, r, m = 2048, 2048, 2, 4
    w_host, w_vals = weights("gauss", n, k, 9, "bf16")
    q, a, z = oracle.quantize_minmax(w_vals)
    packed = gpu_pack(to_dev(q), r)
    x_bits = synth.activations(m, k, 10)
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    wr = oracle.dequant_slice(q, a, z, r)
    for _ in range(3):
        check_linear(gpu_linear(x_bits, packed, to_dev(a), to_dev(z), n, r), x_vals, wr, "repeat")
