"""GPU parity of the Mix'n'Match stack (per-layer widths) against the oracle."""
import numpy as np
import pytest
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import synth
from gpu_util import DEV, check_linear, gpu_pack, gpu_quantize, to_dev, weights

pytestmark = pytest.mark.gpu


def _run_stack(shapes, widths, m, xseed, law="gauss"):
    """shapes: list of (layer, N, K, wseed). Returns (host weights, GPU outputs, inputs)."""
    ks = sorted({k for _, _, k, _ in shapes})
    xs_bits = {k: synth.activations(m, k, xseed + k) for k in ks}
    xs_dev = {k: to_dev(v) for k, v in xs_bits.items()}
    lins, lol, keep, outs = [], [], [], []
    for layer, n, k, seed in shapes:
        w_host, _ = weights(law, n, k, seed, "bf16")
        q, a, z = gpu_quantize(w_host, "bf16")
        packed = gpu_pack(q, widths[layer])
        y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
        keep.append((packed, a, z))
        outs.append(y)
        lins.append((xs_dev[k], packed, a, z, y, n, k))
        lol.append(layer)
        del q
    mq.stack_forward(lins, lol, widths, m)
    mq.device_status()
    return xs_bits, [o.cpu().numpy().astype(np.float64) for o in outs]


@pytest.mark.parametrize("m", [1, 5, 32])
def test_small_stack_all_widths_full_check(m):
    widths = [6, 3, 2, 8, 4]
    shapes = []
    seed = 900
    for layer in range(5):
        for n, k in [(384, 512), (200, 1024), (640, 384)]:
            shapes.append((layer, n, k, seed))
            seed += 1
    xs_bits, outs = _run_stack(shapes, widths, m, 70)
    for (layer, n, k, s), y in zip(shapes, outs):
        _, w_vals = weights("gauss", n, k, s, "bf16")
        q, a, z = oracle.quantize_minmax(w_vals)
        x_vals = synth.f32_from_bf16_bits(xs_bits[k]).astype(np.float64)
        check_linear(y, x_vals, oracle.dequant_slice(q, a, z, widths[layer]), f"layer {layer} {n}x{k}")


def test_7b_shaped_stack_sampled_rows():
    """Four layers of the 7B Mix'n'Match shapes at widths 8, 4, 2, 8; every
    output column checked on 48 sampled weight rows per linear (the oracle
    quantizes rows independently, so a row sample is exact)."""
    widths = [8, 4, 2, 8]
    mats = synth.WORKLOADS["mixnmatch_7b_stack"]["mats"]
    shapes = [(layer, n, k, 1000 + 5 * layer + j) for layer in range(4) for j, (_, n, k) in enumerate(mats)]
    m = 8
    xs_bits, outs = _run_stack(shapes, widths, m, 2000)
    rng = np.random.default_rng(0)
    for (layer, n, k, s), y in zip(shapes, outs):
        assert np.all(np.isfinite(y))
        _, w_vals = weights("gauss", n, k, s, "bf16")
        rows = np.sort(rng.choice(n, size=48, replace=False))
        q, a, z = oracle.quantize_minmax(w_vals[rows])
        x_vals = synth.f32_from_bf16_bits(xs_bits[k]).astype(np.float64)
        check_linear(y[:, rows], x_vals, oracle.dequant_slice(q, a, z, widths[layer]),
                     f"layer {layer} {n}x{k}")
