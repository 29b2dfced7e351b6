"""Short integer decode launches (one batch row, r = 8, 4, 2) that run
without the prep kernel: each CTA's producer warp stages its units' digit
blocks from x, the CTAs zero the row blocks they share and meet at a grid
barrier before adding into them. These tests issue many such launches back
to back on one stream (and from a replayed CUDA graph), with row blocks split
across CTAs and units that fall back to bf16, and compare every output with
the float64 oracle within |y - y_ref| <= 1e-3 sum_k |x||W_r| + 1e-6.
"""
import numpy as np
import pytest
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import synth
from gpu_util import DEV, check_linear, gpu_pack, to_dev

pytestmark = pytest.mark.gpu

# (N, K, r): from one unit to a few per CTA, every row block shared
SHAPES = [(256, 128, 8), (512, 1024, 8), (512, 1024, 4), (512, 1024, 2), (4096, 4096, 4),
          (2304, 2304, 2), (9216, 2304, 8), (300, 4160, 2), (1000, 96, 4)]


def _case(n, k, r, seed, outliers=False):
    w = synth.f32_from_bf16_bits(synth.gaussian_weights(n, k, seed)).astype(np.float64)
    q, a, z = oracle.quantize_minmax(w)
    x_bits = synth.activations(1, k, seed + 1)
    if outliers:
        # inputs 2^-60 next to 1.0 in some units: those units take the bf16 path
        x_bits = x_bits.copy()
        x_bits[0, ::97] = synth.bf16_bits_from_f32(np.float32(2.0 ** -60))
    xv = synth.f32_from_bf16_bits(x_bits).astype(np.float64)
    return dict(n=n, k=k, r=r, packed=gpu_pack(to_dev(q), r), a=to_dev(a), z=to_dev(z), x=to_dev(x_bits),
                xv=xv, wr=oracle.dequant_slice(q, a, z, r))


@pytest.fixture(scope="module")
def cases():
    return [_case(n, k, r, 40 + i, outliers=(i % 3 == 2)) for i, (n, k, r) in enumerate(SHAPES)]


def _run(c, y, stream=None):
    mq.linear(c["x"], 1, c["k"], c["packed"], c["a"], c["z"], c["n"], c["r"], y, stream)


def test_back_to_back_launches(cases):
    rounds = 6
    ys = [[torch.full((1, c["n"]), float("nan"), dtype=torch.float32, device=DEV) for c in cases]
          for _ in range(rounds)]
    for i in range(rounds):
        for c, y in zip(cases, ys[i]):
            _run(c, y)
    mq.device_status()
    for i in range(rounds):
        for c, y in zip(cases, ys[i]):
            check_linear(y.cpu().numpy().astype(np.float64), c["xv"], c["wr"],
                         f"round {i} N={c['n']} K={c['k']} r={c['r']}")


def test_same_output_rewritten(cases):
    """A launch that adds into row blocks must start from zero every time,
    whatever the previous launch left in y."""
    c = cases[4]
    y = torch.full((1, c["n"]), 1e30, dtype=torch.float32, device=DEV)
    for _ in range(10):
        _run(c, y)
    mq.device_status()
    check_linear(y.cpu().numpy().astype(np.float64), c["xv"], c["wr"], "rewritten output")


def test_graph_replays(cases):
    side = torch.cuda.Stream()
    ys = [torch.full((1, c["n"]), float("nan"), dtype=torch.float32, device=DEV) for c in cases]
    with torch.cuda.stream(side):
        for c, y in zip(cases, ys):
            _run(c, y, side)
    side.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for c, y in zip(cases, ys):
            _run(c, y, side)
    for rep in range(5):
        for y in ys:
            y.fill_(float("nan"))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        mq.device_status(side)
        for c, y in zip(cases, ys):
            check_linear(y.cpu().numpy().astype(np.float64), c["xv"], c["wr"],
                         f"replay {rep} N={c['n']} K={c['k']} r={c['r']}")
    del g
    torch.cuda.synchronize()
