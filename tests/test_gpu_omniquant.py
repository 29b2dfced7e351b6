"""GPU parity of Eq. 3 (OmniQuant's clipped MinMax with given per-row gamma,
beta) against the oracle: bit-exact codes, alpha and z on the workloads'
weight shapes, ragged shapes and the range rules; and the clipped container
feeding the packed planes and the decode linear."""
import numpy as np
import pytest
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import synth
from gpu_util import DEV, check_linear, gpu_linear, gpu_pack, gpu_quantize, to_dev, weights

pytestmark = pytest.mark.gpu


def gpu_quantize_clipped(w_host, dtype, gamma, beta):
    n, k = w_host.shape
    w_d = to_dev(w_host)
    g_d = to_dev(np.asarray(gamma, dtype=np.float32))
    b_d = to_dev(np.asarray(beta, dtype=np.float32))
    q = torch.empty((n, k), dtype=torch.uint8, device=DEV)
    a = torch.empty(n, dtype=torch.float32, device=DEV)
    z = torch.empty(n, dtype=torch.float32, device=DEV)
    mq.quantize_int8_clipped(w_d, mq.MQ_F32 if dtype == "f32" else mq.MQ_BF16, n, k, g_d, b_d,
                             q, a, z)
    torch.cuda.synchronize()
    return q, a, z


def _assert_clipped_equal(w_host, w_vals, dtype, gamma, beta):
    q, a, z = gpu_quantize_clipped(w_host, dtype, gamma, beta)
    q_ref, a_ref, z_ref = oracle.quantize_omniquant(w_vals, gamma, beta)
    assert np.array_equal(a.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
    assert np.array_equal(z.cpu().numpy().view(np.uint32), z_ref.view(np.uint32))
    qg = q.cpu().numpy()
    if not np.array_equal(qg, q_ref):
        bad = np.argwhere(qg != q_ref)
        raise AssertionError(f"{len(bad)} codes differ, first {bad[0]}: "
                             f"{qg[tuple(bad[0])]} vs {q_ref[tuple(bad[0])]}")
    return q, a, z, q_ref


@pytest.mark.parametrize("name,law,n,k,seed,dtype", [
    ("single_linear_fp32", "gauss", 512, 1024, 0, "f32"),
    ("gemma2b_gate", "gauss", 9216, 2304, 104, "bf16"),
    ("mistral_up_heavy_tail", "t", 14336, 4096, 300, "bf16"),
    ("mistral_down_heavy_tail", "t", 4096, 14336, 301, "bf16"),
    ("gemma9b_up", "gauss", 14336, 3584, 500, "bf16"),
])
def test_clipped_workload_shapes(name, law, n, k, seed, dtype):
    w_host, w_vals = weights(law, n, k, seed, dtype)
    gamma = synth.clip_factors(n, seed + 1)
    beta = synth.clip_factors(n, seed + 2)
    _, _, _, q_ref = _assert_clipped_equal(w_host, w_vals, dtype, gamma, beta)
    # the factors below 1 really clip: both ends saturate somewhere
    assert (q_ref == 0).sum() > n and (q_ref == 255).sum() > n


@pytest.mark.parametrize("n,k", [(1, 1), (3, 7), (5, 100), (2, 4097), (17, 48)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_clipped_ragged_shapes(n, k, dtype):
    w_host, w_vals = weights("t", n, k, 11 + n + k, dtype)
    _assert_clipped_equal(w_host, w_vals, dtype, synth.clip_factors(n, n), synth.clip_factors(n, k))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_unit_factors_equal_eq1_kernel(dtype):
    # gamma = beta = 1 is Eq. 1: the clipped entry point and mq_quantize_int8
    # give the same bits
    n, k = 4096, 14336
    w_host, w_vals = weights("t", n, k, 77, dtype)
    ones = np.ones(n, dtype=np.float32)
    q, a, z, _ = _assert_clipped_equal(w_host, w_vals, dtype, ones, ones)
    q1, a1, z1 = gpu_quantize(w_host, dtype)
    assert torch.equal(q, q1) and torch.equal(a, a1) and torch.equal(z, z1)


def test_clipped_range_rules():
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((8, 256)) * 0.02).astype(np.float32)
    w[0] = 0.125                      # constant row
    w[1, :] = 0.0                     # all zero
    w[2] = np.abs(w[2]) + 1.0         # all positive: beta * min > 0
    w[3] = -np.abs(w[3]) - 1.0        # all negative
    w[4] *= 1e4
    gamma = np.array([0.9, 0.5, 0.7, 1.0, 0.8, 0.0, 0.3, 1.0], dtype=np.float32)
    beta = np.array([0.9, 0.5, 1.0, 0.7, 0.8, 0.0, 1.0, 0.3], dtype=np.float32)
    # row 5: gamma = beta = 0 (empty range, alpha = 2^-126); rows 6, 7 one-sided clipping
    _assert_clipped_equal(w, w.astype(np.float64), "f32", gamma, beta)
    # inverted range: gamma * max < beta * min for an all-positive row
    w2 = (np.abs(rng.standard_normal((2, 64))) + 2.0).astype(np.float32)
    _assert_clipped_equal(w2, w2.astype(np.float64), "f32", np.array([0.1, 0.2], np.float32),
                          np.array([1.0, 1.0], np.float32))


def test_clipped_container_through_planes_and_linear():
    # quantize with clipping, slice to r = 4 and r = 2, run the decode linear:
    # planes bit-exact with the oracle's, outputs within the stated tolerance
    n, k, m = 4096, 4096, 4
    w_host, w_vals = weights("t", n, k, 900, "bf16")
    gamma, beta = synth.clip_factors(n, 901), synth.clip_factors(n, 902)
    q, a, z, q_ref = _assert_clipped_equal(w_host, w_vals, "bf16", gamma, beta)
    _, a_ref, z_ref = oracle.quantize_omniquant(w_vals, gamma, beta)
    x = synth.activations(m, k, 903)
    x_vals = synth.f32_from_bf16_bits(x).astype(np.float64)
    for r in (4, 2):
        packed = gpu_pack(q, r)
        want = oracle.pack_rows(oracle.slice_codes(q_ref, r), r)
        assert np.array_equal(packed.cpu().numpy()[: mq.packed_bytes(n, k, r)], want)
        w_r = oracle.dequant_slice(q_ref, a_ref, z_ref, r)
        y = gpu_linear(x, packed, a, z, n, r)
        check_linear(y, x_vals, w_r, f"clipped r={r}")
