"""GPU parity of the chained decoder stack (mq_chain_forward) against the
float64 oracle chain with the same stand-in glue.

Tolerance. Each linear of the decode path stays within 1e-3 sum_k |x||W|
per output. The residual stream collects, per layer, the errors of the `o`
and `down` linears directly; the errors of qkv, gate and up reach it
through those two linears' inputs (scaled by the same |W| sums), and a bf16
rounding of a linear input that lands on the other side of a boundary than
the oracle's float64 value moves one element by one bf16 step, which adds
less again. So every element of h must agree with the oracle within 3 times
the running sum over the layers of 1e-3 (|a| |W_o|^T + |act| |W_down|^T),
computed by the oracle (plus 1e-6). A dropped term, a wrong head-to-group
map or a missing residual misses by far more."""
import numpy as np
import pytest
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import oracle.chain as och
import synth
from gpu_util import DEV, gpu_pack, to_dev

pytestmark = pytest.mark.gpu


def build_chain(n_layers, widths, D, Dkv, F, seed):
    """Per layer: the oracle's dequantized W_r for each linear (float64) and
    the device tensors (packed planes at the layer's width, alpha, zero)."""
    shapes = [(D + 2 * Dkv, D), (D, D), (F, D), (F, D), (D, F)]
    names = ["qkv", "o", "gate", "up", "down"]
    ref_layers, dev_layers, keep = [], [], []
    for l in range(n_layers):
        r = widths[l]
        ref, lins = {}, []
        for i, (n, k) in enumerate(shapes):
            w = synth.f32_from_bf16_bits(synth.gaussian_weights(n, k, seed + 10 * l + i)).astype(np.float64)
            q, a, z = oracle.quantize_minmax(w)
            ref[names[i]] = oracle.dequant_slice(q, a, z, r)
            p, ad, zd = gpu_pack(to_dev(q), r), to_dev(a), to_dev(z)
            keep += [p, ad, zd]
            lins.append((p, ad, zd))
        ref_layers.append(ref)
        dev_layers.append((r, lins))
    return ref_layers, dev_layers, keep


def run_gpu(dev_layers, h0, M, D, Dkv, F, hd, graph=False, stream=None):
    plan = mq.ChainPlan(dev_layers, M, D, Dkv, F, hd)
    scratch = torch.empty(mq.chain_scratch_bytes(M, D, Dkv, F), dtype=torch.uint8, device=DEV)
    h = torch.from_numpy(h0.astype(np.float32)).to(DEV)
    plan.run(h, scratch, graph=graph, stream=stream)
    mq.device_status(stream)
    return h.cpu().numpy().astype(np.float64)


def check(h_gpu, h_ref, bound, label):
    tol = 3.0 * bound + 1e-6
    err = np.abs(h_gpu - h_ref)
    assert np.all(np.isfinite(h_gpu)), label
    ratio = err / tol
    assert ratio.max() <= 1.0, f"{label}: err/tol {ratio.max():.3g} at {np.unravel_index(ratio.argmax(), ratio.shape)}"
    return ratio.max()


@pytest.mark.parametrize("M", [1, 3])
def test_chain_small_every_depth(M):
    D, Dkv, F, hd = 512, 128, 1024, 64
    widths = [8, 4, 2, 3, 6]
    ref_layers, dev_layers, _keep = build_chain(5, widths, D, Dkv, F, 100)
    h0 = np.random.default_rng(M).standard_normal((M, D))
    trace, bound = [], []
    och.chain_forward(h0, ref_layers, D, Dkv, hd, trace=trace, bound=bound)
    for depth in range(1, 6):
        h = run_gpu(dev_layers[:depth], h0, M, D, Dkv, F, hd)
        print(f"depth {depth} M={M} err/tol {check(h, trace[depth - 1], bound[depth - 1], f'depth {depth} M={M}'):.3f}")


def test_chain_7b_shapes_two_layers():
    D, Dkv, F, hd, M = 4096, 1024, 14336, 128, 1
    ref_layers, dev_layers, _keep = build_chain(2, [8, 2], D, Dkv, F, 200)
    h0 = np.random.default_rng(7).standard_normal((M, D))
    bound = []
    h_ref = och.chain_forward(h0, ref_layers, D, Dkv, hd, bound=bound)
    r = check(run_gpu(dev_layers, h0, M, D, Dkv, F, hd), h_ref, bound[-1], "7B shapes")
    print(f"7B shapes err/tol {r:.3f}")


def test_chain_graph_replay_matches_direct():
    # first call direct, second captured and launched, third replayed: all
    # three agree with the oracle, and with each other to rounding
    D, Dkv, F, hd, M = 512, 128, 1024, 64, 2
    ref_layers, dev_layers, _keep = build_chain(3, [4, 2, 8], D, Dkv, F, 300)
    h0 = np.random.default_rng(9).standard_normal((M, D))
    bound = []
    h_ref = och.chain_forward(h0, ref_layers, D, Dkv, hd, bound=bound)
    plan = mq.ChainPlan(dev_layers, M, D, Dkv, F, hd)
    scratch = torch.empty(mq.chain_scratch_bytes(M, D, Dkv, F), dtype=torch.uint8, device=DEV)
    h = torch.empty((M, D), dtype=torch.float32, device=DEV)
    s = torch.cuda.Stream()
    outs = []
    for _ in range(4):
        with torch.cuda.stream(s):
            h.copy_(torch.from_numpy(h0.astype(np.float32)))
            plan.run(h, scratch, graph=True, stream=s)
        s.synchronize()
        mq.device_status(s)
        outs.append(h.cpu().numpy().astype(np.float64))
    for i, o in enumerate(outs):
        check(o, h_ref, bound[-1], f"call {i}")
    tol = 1e-5 * np.sqrt(np.mean(h_ref * h_ref))
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= tol
    mq.release_workspace()


def test_chain_rejects_bad_arguments():
    D, Dkv, F, hd, M = 512, 128, 1024, 64, 1
    _, dev_layers, _keep = build_chain(1, [4], D, Dkv, F, 400)
    plan = mq.ChainPlan(dev_layers, M, D, Dkv, F, hd)
    small = torch.empty(256, dtype=torch.uint8, device=DEV)
    h = torch.zeros((M, D), dtype=torch.float32, device=DEV)
    with pytest.raises(mq.MQError):
        plan.run(h, small)
    bad = mq.ChainPlan(dev_layers, M, D, Dkv, F, 48)   # head_dim does not divide Dkv
    scratch = torch.empty(mq.chain_scratch_bytes(M, D, Dkv, F), dtype=torch.uint8, device=DEV)
    with pytest.raises(mq.MQError):
        bad.run(h, scratch)
