"""GPU parity of the prefill GEMM (M > 32, tensor cores with accumulators in
tensor memory) against the float64 oracle, element by element within
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


def _case(law, n, k, seed, r, m, xseed, rows=None):
    w_host, w_vals = weights(law, n, k, seed, "bf16")
    q, a, z = oracle.quantize_minmax(w_vals)
    packed = gpu_pack(to_dev(q), r)
    x_bits = synth.activations(m, k, xseed)
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    y = gpu_linear(x_bits, packed, to_dev(a), to_dev(z), n, r)
    if rows is None:
        return check_linear(y, x_vals, oracle.dequant_slice(q, a, z, r), f"{law} {n}x{k} r={r} M={m}")
    # rows are quantized independently, so the oracle on a row sample is exact
    return check_linear(y[:, rows], x_vals, oracle.dequant_slice(q[rows], a[rows], z[rows], r),
                        f"{law} {n}x{k} r={r} M={m} (sampled rows)")


@pytest.mark.parametrize("r", WIDTHS)
@pytest.mark.parametrize("m", [33, 64, 128, 129, 200])
def test_all_widths_ragged_batches(r, m):
    _case("gauss", 256, 512, 20 + r, r, m, 30 + m)


@pytest.mark.parametrize("r", WIDTHS)
@pytest.mark.parametrize("n,k", [(1, 128), (127, 256), (129, 384), (300, 1152), (1000, 896)])
def test_ragged_weight_shapes(r, n, k):
    _case("t", n, k, n + k, r, 77, n)


@pytest.mark.parametrize("r", [6, 4, 3, 2])
@pytest.mark.parametrize("name,n,k,seed", [("up", 14336, 3584, 500), ("down", 3584, 14336, 501)])
def test_gemma9b_prefill_sampled_rows(name, n, k, seed, r):
    """The 9B-shaped prefill matrices at M = 2048: every batch row of 64
    sampled weight rows (spread over every 128-row tile boundary region)."""
    rng = np.random.default_rng(seed + r)
    rows = np.unique(np.concatenate([rng.choice(n, size=48, replace=False), [0, 127, 128, n - 1]]))
    _case("gauss", n, k, seed, r, 2048, 600, rows=rows)


@pytest.mark.parametrize("r", [8, 4, 2])
def test_heavy_tail_mistral_shape(r):
    rng = np.random.default_rng(r)
    rows = np.sort(rng.choice(4096, size=64, replace=False))
    _case("t", 4096, 14336, 301, r, 96, 401, rows=rows)


def test_gemm_matches_decode_at_the_boundary():
    """M = 32 runs the decode GEMV and M = 33 the GEMM: the first 32 rows of
    the two results must agree within the tolerance."""
    n, k, r = 640, 1024, 4
    w_host, w_vals = weights("gauss", n, k, 3, "bf16")
    q, a, z = oracle.quantize_minmax(w_vals)
    packed = gpu_pack(to_dev(q), r)
    x_bits = synth.activations(33, k, 4)
    y33 = gpu_linear(x_bits, packed, to_dev(a), to_dev(z), n, r)
    y32 = gpu_linear(x_bits[:32], packed, to_dev(a), to_dev(z), n, r)
    x_vals = synth.f32_from_bf16_bits(x_bits[:32]).astype(np.float64)
    tol = oracle.tolerance(x_vals, oracle.dequant_slice(q, a, z, r))
    assert np.all(np.abs(y33[:32] - y32) <= 2 * tol)


def test_gemm_timeout_path_reports_and_recovers():
    n, k, r, m = 512, 1024, 4, 256
    w_host, w_vals = weights("gauss", n, k, 1, "bf16")
    q, a, z = oracle.quantize_minmax(w_vals)
    packed = gpu_pack(to_dev(q), r)
    x_bits = synth.activations(m, k, 2)
    x_d = to_dev(x_bits)
    y = torch.zeros((m, n), dtype=torch.float32, device=DEV)
    mq.debug_set_wait_limit_ns(0)
    try:
        mq.linear(x_d, m, k, packed, to_dev(a), to_dev(z), n, r, y)
        with pytest.raises(mq.MQError) as e:
            mq.device_status()
        assert e.value.status == mq.MQ_ERR_TIMEOUT
    finally:
        mq.debug_set_wait_limit_ns(2_000_000_000)
    mq.device_status()
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    y2 = gpu_linear(x_bits, packed, to_dev(a), to_dev(z), n, r)
    check_linear(y2, x_vals, oracle.dequant_slice(q, a, z, r), "after timeout")
