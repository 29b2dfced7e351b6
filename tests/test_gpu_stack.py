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


def test_bench_workload_every_linear_sampled_rows():
    """The benchmark's own configuration, in its own launch: the 32-layer
    7B-shaped Mix'n'Match stack (160 linears, widths 8 / 4 / 2 by layer) at
    one batch row, built and stepped by bench.Stack exactly as the timed loop
    does. Every output must be written; on 24 sampled weight rows of every
    linear (first, last and random rows, so both whole and CTA-shared row
    blocks are hit) y must match the oracle, which quantizes the same rows of
    the same seeded weights on the host."""
    import bench
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stack = bench.Stack(1, dev)
    assert len(stack.lins) == 160 and stack.widths == synth.mixnmatch_widths(32)
    stack.y_all.fill_(float("nan"))
    s = torch.cuda.current_stream(dev)
    stack.step(s)
    torch.cuda.synchronize()
    mq.device_status()
    assert bool(torch.isfinite(stack.y_all).all()), "an output element was not written"
    xs = {k: synth.f32_from_bf16_bits(v.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
          for k, v in stack.x.items()}
    rng = np.random.default_rng(5)
    mats = synth.WORKLOADS["mixnmatch_7b_stack"]["mats"]
    worst = 0.0
    for i, (x, p, a, z, y, n, k) in enumerate(stack.lins):
        layer, j = divmod(i, len(mats))
        w = synth.device_gaussian_weights(n, k, stack.seed_base + 5 * layer + j, dev)
        rows = np.unique(np.concatenate([[0, n - 1], rng.choice(n, size=22, replace=False)]))
        w_rows = w[torch.from_numpy(rows).to(dev)].view(torch.int16).cpu().numpy().view(np.uint16)
        q, a_r, z_r = oracle.quantize_minmax(synth.f32_from_bf16_bits(w_rows).astype(np.float64))
        y_rows = y[:, torch.from_numpy(rows).to(dev)].cpu().numpy().astype(np.float64)
        worst = max(worst, check_linear(y_rows, xs[k], oracle.dequant_slice(q, a_r, z_r, stack.widths[layer]),
                                        f"bench stack linear {i} (layer {layer}) {n}x{k}"))
    print(f"bench workload: worst err/tol {worst:.3f}")
