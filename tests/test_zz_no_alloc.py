"""mq_linear_noalloc: the decode GEMV for callers that cannot allocate device
memory (an engine whose allocator owns all of HBM, a plugin that may not
allocate, a decode loop that cannot afford an allocation's synchronization).

It must give the same results as mq_linear, within the tolerance every parity
test here uses (|dy| <= 1e-3 sum_k |x||W_r| + 1e-6), on consecutive calls that
share its one fixed device array. This file is named so that pytest collects it
last.
"""
import numpy as np
import pytest
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import synth


def _tolerance(x_bits, q, a, z, r):
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    return oracle.tolerance(x_vals, oracle.dequant_slice(q, a, z, r))


def test_noalloc_rejects_oversized_calls_on_the_host():
    """Sizes beyond the fixed array are refused before any CUDA call."""
    F = 1 << 20
    st = mq.raw_status("mq_linear_noalloc", F, 32, 32768, F, F, F, 64, 4, F, None)
    assert st == mq.MQ_ERR_INVALID_ARG
    assert "scratch" in mq.last_error()
    # one batch row at r = 2 stages seven digits per input (3648 bytes per 512):
    # K = 183808 is the largest that fits (run on the GPU below), one unit more
    # is refused; at r = 4 (1856 bytes per 256) K = 180480 fits, 180736 not
    assert mq.raw_status("mq_linear_noalloc", F, 1, 183808 + 512, F, F, F, 64, 2, F, None) == mq.MQ_ERR_INVALID_ARG
    assert "scratch" in mq.last_error()
    assert mq.raw_status("mq_linear_noalloc", F, 1, 180480 + 256, F, F, F, 64, 4, F, None) == mq.MQ_ERR_INVALID_ARG
    assert "scratch" in mq.last_error()
    # two batch rows at r = 4 stage bf16 (two bytes per input): M K = 2 x 327424 fits, 2 x 327680 not
    assert mq.raw_status("mq_linear_noalloc", F, 2, 327680, F, F, F, 64, 4, F, None) == mq.MQ_ERR_INVALID_ARG
    assert "scratch" in mq.last_error()
    assert mq.raw_status("mq_linear_noalloc", F, 33, 256, F, F, F, 64, 4, F, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_linear_noalloc", F, 1, 256, F, F, F, 64, 5, F, None) == mq.MQ_ERR_INVALID_ARG


@pytest.mark.gpu
def test_noalloc_matches_linear_on_consecutive_calls():
    dev = "cuda:0"
    torch.cuda.set_device(0)

    def up(a):
        a = np.ascontiguousarray(a)
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(dev)

    # (M, N, K, r, weight seed): the second call is the largest M * K the
    # fixed array serves, with another width and shape, so it reuses the
    # array after the first call left its own contents there. The last two
    # are r = 2 at one batch row (inputs staged as integer digits), the
    # largest K of that layout last; then K a multiple of 32 or 64 only.
    cases = [(8, 2048, 4096, 4, 31), (32, 1000, 16384, 2, 32), (1, 777, 2304, 8, 33),
             (1, 1500, 8192, 2, 34), (1, 64, 183808, 2, 35),
             (1, 300, 96, 4, 36), (3, 200, 4160, 2, 37)]   # K on the width's own unit (32, 64)
    for M, N, K, r, seed in cases:
        w = synth.f32_from_bf16_bits(synth.gaussian_weights(N, K, seed)).astype(np.float64)
        q, a, z = oracle.quantize_minmax(w)
        x_bits = synth.activations(M, K, seed + 100)
        x, a_d, z_d = up(x_bits), up(a), up(z)
        packed = torch.empty(mq.packed_bytes(N, K, r), dtype=torch.uint8, device=dev)
        mq.slice_pack(up(q), N, K, r, packed)

        y_lin = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
        mq.linear(x, M, K, packed, a_d, z_d, N, r, y_lin)
        y_na = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
        mq.linear_noalloc(x, M, K, packed, a_d, z_d, N, r, y_na)
        torch.cuda.synchronize()
        mq.device_status()

        y1 = y_lin.cpu().numpy().astype(np.float64)
        y2 = y_na.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(y2)), f"M={M} N={N} K={K} r={r}: unwritten output"
        tol = _tolerance(x_bits, q, a, z, r)
        err = np.abs(y2 - y1)
        assert np.all(err <= tol), (
            f"M={M} N={N} K={K} r={r}: {int((err > tol).sum())} elements differ from mq_linear "
            f"beyond the tolerance (max ratio {float((err / tol).max()):.3g})")
        # and against the float64 oracle itself, so a fault the two entry
        # points share cannot pass
        x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
        y_ref = oracle.linear(x_vals, oracle.dequant_slice(q, a, z, r))
        err = np.abs(y2 - y_ref)
        assert np.all(err <= tol), (
            f"M={M} N={N} K={K} r={r}: {int((err > tol).sum())} elements outside the tolerance "
            f"of the oracle (max ratio {float((err / tol).max()):.3g})")


@pytest.mark.gpu
def test_noalloc_timeout_is_reported_and_recovers():
    """A wait limit of 0 makes every pipeline wait of the call give up at
    once. The give-up lands in the fixed array's error word, which
    mq_device_status() must report as MQ_ERR_TIMEOUT (and clear); the next
    call must then be correct."""
    dev = "cuda:0"
    torch.cuda.set_device(0)
    M, N, K, r = 1, 640, 2048, 2
    w = synth.f32_from_bf16_bits(synth.gaussian_weights(N, K, 36)).astype(np.float64)
    q, a, z = oracle.quantize_minmax(w)
    x_bits = synth.activations(M, K, 136)

    def up(v):
        v = np.ascontiguousarray(v)
        return torch.from_numpy(v.view(np.int16) if v.dtype == np.uint16 else v).to(dev)

    x, a_d, z_d = up(x_bits), up(a), up(z)
    packed = torch.empty(mq.packed_bytes(N, K, r), dtype=torch.uint8, device=dev)
    mq.slice_pack(up(q), N, K, r, packed)
    y = torch.zeros((M, N), dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    mq.device_status()
    mq.debug_set_wait_limit_ns(0)
    try:
        mq.linear_noalloc(x, M, K, packed, a_d, z_d, N, r, y)
        with pytest.raises(mq.MQError) as e:
            mq.device_status()
        assert e.value.status == mq.MQ_ERR_TIMEOUT
    finally:
        mq.debug_set_wait_limit_ns(2_000_000_000)
    mq.device_status()  # the flag was cleared
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
    mq.linear_noalloc(x, M, K, packed, a_d, z_d, N, r, y)
    mq.device_status()
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    wr = oracle.dequant_slice(q, a, z, r)
    err = np.abs(y.cpu().numpy().astype(np.float64) - oracle.linear(x_vals, wr))
    assert np.all(err <= oracle.tolerance(x_vals, wr))
