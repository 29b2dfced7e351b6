"""GPU parity of Eq. 1 (int8 container) and Eq. 6 packed planes against the
oracle: bit-exact on the workloads' weight shapes and on edge cases."""
import numpy as np
import pytest
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import synth
from gpu_util import DEV, gpu_pack, gpu_quantize, to_dev, weights

pytestmark = pytest.mark.gpu

WIDTHS = [8, 6, 4, 3, 2]


def _assert_quant_equal(w_host, w_vals, dtype):
    q, a, z = gpu_quantize(w_host, dtype)
    q_ref, a_ref, z_ref = oracle.quantize_minmax(w_vals)
    assert np.array_equal(a.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
    assert np.array_equal(z.cpu().numpy().view(np.uint32), z_ref.view(np.uint32))
    qg = q.cpu().numpy()
    if not np.array_equal(qg, q_ref):
        bad = np.argwhere(qg != q_ref)
        raise AssertionError(f"{len(bad)} codes differ, first {bad[0]}: {qg[tuple(bad[0])]} vs {q_ref[tuple(bad[0])]}")
    return q_ref, a_ref, z_ref


@pytest.mark.parametrize("name,law,n,k,seed,dtype", [
    ("single_linear_fp32", "gauss", 512, 1024, 0, "f32"),
    ("gemma2b_qkvo", "gauss", 2304, 2304, 100, "bf16"),
    ("gemma2b_gate", "gauss", 9216, 2304, 104, "bf16"),
    ("gemma2b_down", "gauss", 2304, 9216, 106, "bf16"),
    ("mistral_up_heavy_tail", "t", 14336, 4096, 300, "bf16"),
    ("mistral_down_heavy_tail", "t", 4096, 14336, 301, "bf16"),
    ("gemma9b_up", "gauss", 14336, 3584, 500, "bf16"),
])
def test_quantize_workload_shapes(name, law, n, k, seed, dtype):
    w_host, w_vals = weights(law, n, k, seed, dtype)
    _assert_quant_equal(w_host, w_vals, dtype)


@pytest.mark.parametrize("n,k", [(1, 1), (3, 7), (5, 100), (2, 4097), (17, 48)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_ragged_shapes(n, k, dtype):
    w_host, w_vals = weights("gauss", n, k, 7 + n + k, dtype)
    _assert_quant_equal(w_host, w_vals, dtype)


def test_quantize_degenerate_and_extreme_rows():
    rng = np.random.default_rng(0)
    w = (rng.standard_normal((6, 256)) * 0.02).astype(np.float32)
    w[0] = 0.125                      # constant row
    w[1] = -3.0                       # constant negative row
    w[2, :] = 0.0
    w[2, 7] = 1e-30                   # tiny range
    w[3] *= 1e4                       # large range
    w[4] = np.abs(w[4]) + 100.0       # far from zero (z < 0, cancellation in w/alpha + z)
    w[5, ::2] = 0.5
    w[5, 1::2] = -0.5                 # only two values
    _assert_quant_equal(w, w.astype(np.float64), "f32")


# the K a width packs: every plane row a whole number of 16-byte units
K_UNIT = {8: 32, 4: 32, 6: 64, 2: 64, 3: 128}


@pytest.mark.parametrize("r", WIDTHS)
@pytest.mark.parametrize("n,k", [(1, 1), (3, 2), (5, 3), (129, 256), (2304, 2304), (4096, 14336)])
def test_slice_pack_bit_exact(r, n, k):
    if k <= 3:
        k *= K_UNIT[r]  # one, two and three of the width's K units
    rng = np.random.default_rng(n * 31 + k + r)
    q = rng.integers(0, 256, size=(n, k), dtype=np.uint8)
    q[:, 0] = 0
    q[:, -1] = 255
    packed = gpu_pack(to_dev(q), r).cpu().numpy()[: mq.packed_bytes(n, k, r)]
    want = oracle.pack_rows(oracle.slice_codes(q, r), r)
    assert np.array_equal(packed, want)


@pytest.mark.parametrize("r", WIDTHS)
def test_slice_table_all_256_values(r):
    # one row holding every container value, 8 times over: the GPU slice of
    # each q equals the oracle's brute-force table
    q = np.tile(np.arange(256, dtype=np.uint8), 8)[None, :]
    packed = gpu_pack(to_dev(q), r).cpu().numpy()[: mq.packed_bytes(1, q.shape[1], r)]
    codes = oracle.unpack_rows(packed, 1, q.shape[1], r)[0]
    assert np.array_equal(codes[:256], oracle.slice_table(r))


def test_full_width_pack_is_container():
    q = np.random.default_rng(3).integers(0, 256, size=(64, 512), dtype=np.uint8)
    packed = gpu_pack(to_dev(q), 8).cpu().numpy()[: q.size]
    assert np.array_equal(packed, q.reshape(-1))


def test_repeated_runs_identical():
    w_host, _ = weights("t", 1024, 2048, 42, "bf16")
    q1, a1, z1 = gpu_quantize(w_host, "bf16")
    q2, a2, z2 = gpu_quantize(w_host, "bf16")
    assert torch.equal(q1, q2) and torch.equal(a1, a2) and torch.equal(z1, z2)
    for r in WIDTHS:
        assert torch.equal(gpu_pack(q1, r), gpu_pack(q1, r))
