"""GPU parity of Extra Precision on the planes (the errata section's Eq. 8):
the sparse list of extra-bucket positions (bit-exact against the oracle's
Eq. 8 vs Eq. 6 codes) and the decode product from the Eq. 6 planes plus the
list (within |y - y_ref| <= 1e-3 sum_k |x||W_8| + 1e-6 against the float64
oracle with the unclamped codes)."""
import numpy as np
import pytest
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import synth
from gpu_util import DEV, check_linear, gpu_pack, to_dev

pytestmark = pytest.mark.gpu


def _weights(n, k, seed, frac=0.025):
    w = synth.f32_from_bf16_bits(synth.extra_bucket_weights(n, k, seed, frac=frac))
    return w.astype(np.float64)


def oracle_list(q, r):
    """Row offsets and columns of the positions whose unclamped (Eq. 8) code
    differs from the clamped (Eq. 6) one."""
    diff = oracle.slice_codes(q, r, clamp=False) != oracle.slice_codes(q, r)
    counts = diff.sum(axis=1)
    rows = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    cols = np.nonzero(diff)[1].astype(np.uint16)  # row-major order: increasing within a row
    return rows, cols


def gpu_list(q_dev, n, k, r):
    rows = torch.full((n + 1,), -7, dtype=torch.int32, device=DEV)
    mq.ep_overflow_rows(q_dev, n, k, r, rows)
    total = int(rows[n].item())
    cols = torch.empty(max(total, 8), dtype=torch.int16, device=DEV)
    mq.ep_overflow_cols(q_dev, n, k, r, rows, cols)
    torch.cuda.synchronize()
    return rows, cols, total


@pytest.mark.parametrize("r", [6, 4, 3, 2])
@pytest.mark.parametrize("n,k,seed", [(14336, 4096, 300), (4096, 14336, 301), (1, 16, 3),
                                      (3, 48, 4), (1000, 528, 5), (77, 65536, 6)])
def test_overflow_list_bit_exact(r, n, k, seed):
    q, _, _ = oracle.quantize_minmax(_weights(n, k, seed))
    rows, cols, total = gpu_list(to_dev(q), n, k, r)
    want_rows, want_cols = oracle_list(q, r)
    assert np.array_equal(rows.cpu().numpy(), want_rows)
    assert total == len(want_cols)
    assert np.array_equal(cols.cpu().numpy().view(np.uint16)[:total], want_cols)


def test_overflow_list_every_byte():
    # rows of every container value: the list holds exactly q >= 256 - 2^(7-r)
    q = np.tile(np.arange(256, dtype=np.uint8), (5, 4))
    for r in (6, 4, 3, 2):
        rows, cols, total = gpu_list(to_dev(q), 5, 1024, r)
        want_rows, want_cols = oracle_list(q, r)
        assert np.array_equal(rows.cpu().numpy(), want_rows)
        assert np.array_equal(cols.cpu().numpy().view(np.uint16)[:total], want_cols)
        assert total == 5 * 4 * 2 ** (7 - r)


def _ep_case(n, k, seed, r, m, xseed, frac=0.025):
    w = _weights(n, k, seed, frac)
    q, a, z = oracle.quantize_minmax(w)
    q_dev = to_dev(q)
    packed = gpu_pack(q_dev, r)
    rows, cols, _ = gpu_list(q_dev, n, k, r)
    x_bits = synth.activations(m, k, xseed)
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    mq.linear_ep(to_dev(x_bits), m, k, packed, to_dev(a), to_dev(z), n, r, rows, cols, y)
    mq.device_status()
    w8 = oracle.dequant_slice(q, a, z, r, clamp=False)
    return check_linear(y.cpu().numpy().astype(np.float64), x_vals, w8,
                        f"ep {n}x{k} r={r} M={m}")


@pytest.mark.parametrize("r", [6, 4, 3, 2])
@pytest.mark.parametrize("m", [1, 2, 3, 8, 32])
def test_linear_ep_mistral_up(r, m):
    _ep_case(14336, 4096, 300, r, m, 500 + m)


@pytest.mark.parametrize("m", [1, 5])
@pytest.mark.parametrize("n,k", [(1, 128), (257, 640), (4096, 14336), (130, 4224)])
def test_linear_ep_shapes(n, k, m):
    _ep_case(n, k, 17 + n, 2, m, 19 + k)


def test_linear_ep_dense_bucket():
    # half of every row in the extra bucket: the sparse sums carry real weight
    _ep_case(2048, 4096, 40, 2, 1, 41, frac=0.5)
    _ep_case(2048, 4096, 42, 2, 4, 43, frac=0.5)


def test_linear_ep_empty_list_is_eq6():
    # no position in the extra bucket: the result is the planes' product. Row
    # blocks that two CTAs share are summed with fp32 atomics in either order,
    # so the two calls agree to rounding, far inside the tolerance
    n, k, r, m = 4096, 4096, 2, 3
    rng = np.random.default_rng(9)
    q = rng.integers(0, 224, size=(n, k), dtype=np.uint8)
    a = (rng.uniform(0.5, 2.0, n) * 1e-3).astype(np.float32)
    z = rng.uniform(0.0, 255.0, n).astype(np.float32)
    q_dev = to_dev(q)
    packed = gpu_pack(q_dev, r)
    rows, cols, total = gpu_list(q_dev, n, k, r)
    assert total == 0
    x = to_dev(synth.activations(m, k, 10))
    y1 = torch.empty((m, n), dtype=torch.float32, device=DEV)
    y2 = torch.empty((m, n), dtype=torch.float32, device=DEV)
    mq.linear(x, m, k, packed, to_dev(a), to_dev(z), n, r, y1)
    mq.linear_ep(x, m, k, packed, to_dev(a), to_dev(z), n, r, rows, cols, y2)
    torch.cuda.synchronize()
    x_vals = synth.f32_from_bf16_bits(synth.activations(m, k, 10)).astype(np.float64)
    w6 = oracle.dequant_slice(q, a, z, r)
    check_linear(y2.cpu().numpy().astype(np.float64), x_vals, w6, "ep with an empty list")
    tol = oracle.tolerance(x_vals, w6)
    assert np.all(np.abs(y1.cpu().numpy() - y2.cpu().numpy()) <= 1e-2 * tol)


def test_linear_ep_agrees_with_container_eq8():
    # Eq. 8 two ways: planes + sparse list, and the container sliced on load
    n, k, r, m = 4096, 4096, 2, 2
    w = _weights(n, k, 50)
    q, a, z = oracle.quantize_minmax(w)
    q_dev = to_dev(q)
    packed = gpu_pack(q_dev, r)
    rows, cols, _ = gpu_list(q_dev, n, k, r)
    x_bits = synth.activations(m, k, 51)
    x = to_dev(x_bits)
    y1 = torch.empty((m, n), dtype=torch.float32, device=DEV)
    y2 = torch.empty((m, n), dtype=torch.float32, device=DEV)
    mq.linear_ep(x, m, k, packed, to_dev(a), to_dev(z), n, r, rows, cols, y1)
    mq.linear_container(x, m, k, q_dev, to_dev(a), to_dev(z), n, r, False, y2)
    torch.cuda.synchronize()
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    tol = oracle.tolerance(x_vals, oracle.dequant_slice(q, a, z, r, clamp=False))
    assert np.all(np.abs(y1.cpu().numpy() - y2.cpu().numpy()) <= 2 * tol)


# Prefill (M > 32): the list goes through a bit plane into the tcgen05 GEMM,
# whose decode adds one step to every listed code.
@pytest.mark.parametrize("r", [6, 4, 3, 2])
@pytest.mark.parametrize("m", [33, 300])
def test_linear_ep_prefill(r, m):
    _ep_case(2048, 4096, 60 + r, r, m, 600 + m)


@pytest.mark.parametrize("n,k,r,m", [(14336, 4096, 2, 40), (130, 4224, 2, 64), (257, 4128, 4, 70),
                                     (300, 192, 6, 33), (1000, 384, 3, 257)])
def test_linear_ep_prefill_shapes(n, k, r, m):
    # K = 4128 at r = 4 ends halfway through a 64-code stage: the half past K
    # has no bit-plane word and adds nothing
    _ep_case(n, k, 70 + n, r, m, 71 + k)


def test_linear_ep_prefill_dense_bucket():
    _ep_case(2048, 4096, 44, 2, 96, 45, frac=0.5)


def test_linear_ep_prefill_agrees_with_container_eq8():
    n, k, r, m = 4096, 4096, 2, 64
    w = _weights(n, k, 52)
    q, a, z = oracle.quantize_minmax(w)
    q_dev = to_dev(q)
    packed = gpu_pack(q_dev, r)
    rows, cols, _ = gpu_list(q_dev, n, k, r)
    x_bits = synth.activations(m, k, 53)
    x = to_dev(x_bits)
    y1 = torch.empty((m, n), dtype=torch.float32, device=DEV)
    y2 = torch.empty((m, n), dtype=torch.float32, device=DEV)
    mq.linear_ep(x, m, k, packed, to_dev(a), to_dev(z), n, r, rows, cols, y1)
    mq.linear_container(x, m, k, q_dev, to_dev(a), to_dev(z), n, r, False, y2)
    torch.cuda.synchronize()
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    w8 = oracle.dequant_slice(q, a, z, r, clamp=False)
    check_linear(y1.cpu().numpy().astype(np.float64), x_vals, w8, "prefill ep, planes + list")
    check_linear(y2.cpu().numpy().astype(np.float64), x_vals, w8, "prefill ep, container")


@pytest.mark.parametrize("r", [4, 2])
def test_linear_ep_prefill_9b_up_sampled_rows(r):
    """The 9B-shaped `up` matrix at M = 2048 from the planes plus the list;
    rows are quantized independently, so the oracle on a row sample is exact."""
    n, k, m = 14336, 3584, 2048
    w = _weights(n, k, 80 + r)
    q, a, z = oracle.quantize_minmax(w)
    q_dev = to_dev(q)
    packed = gpu_pack(q_dev, r)
    rows_l, cols_l, total = gpu_list(q_dev, n, k, r)
    assert total > 0
    x_bits = synth.activations(m, k, 90 + r)
    x_vals = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    mq.linear_ep(to_dev(x_bits), m, k, packed, to_dev(a), to_dev(z), n, r, rows_l, cols_l, y)
    mq.device_status()
    rng = np.random.default_rng(r)
    rows = np.unique(np.concatenate([rng.choice(n, size=48, replace=False), [0, 127, 128, n - 1]]))
    y_rows = y.cpu().numpy()[:, rows].astype(np.float64)
    check_linear(y_rows, x_vals, oracle.dequant_slice(q[rows], a[rows], z[rows], r, clamp=False),
                 f"prefill ep 9B up r={r} M={m} (sampled rows)")
