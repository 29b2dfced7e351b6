"""GPU parity of the chained decoder stack (mq_chain_forward), step by step.

The chain is checked on its own intermediate values, which the call leaves in
the caller's scratch for its last layer (mq_chain_scratch_views): every linear
(qkv, o, gate, up, down) against the float64 oracle on the exact bf16 input
the GPU fed it, within the stated per-linear bound 1e-3 sum_k |x||W| + 1e-6;
the attention gather and the two residual adds exactly (they are a copy with
one bf16 rounding and single fp32 additions); the RMSNorms and SwiGLU within
the bf16 rounding of an fp32 evaluation (oracle.chain's rmsnorm_f32_error and
swiglu_f32_error, through bf16_flip). Running the chain to every depth checks
every layer that way. A propagated end-to-end bound is no use here: the
per-linear bound is a few percent of a typical output at these widths, and a
worst case carried through RMSNorm and SwiGLU grows without limit; the end
result is still compared with the oracle chain as a sanity check on the
composition (relative RMS deviation)."""
import numpy as np
import pytest
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import oracle.chain as och
import synth
from gpu_util import DEV, check_linear, gpu_pack, to_dev

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


def run_gpu(dev_layers, h0, M, D, Dkv, F, hd, graph=False, stream=None, views=False):
    plan = mq.ChainPlan(dev_layers, M, D, Dkv, F, hd)
    scratch = torch.empty(mq.chain_scratch_bytes(M, D, Dkv, F), dtype=torch.uint8, device=DEV)
    h = torch.from_numpy(h0.astype(np.float32)).to(DEV)
    plan.run(h, scratch, graph=graph, stream=stream)
    mq.device_status(stream)
    out = h.cpu().numpy().astype(np.float64)
    if not views:
        return out
    return out, _read_views(scratch, M, D, Dkv, F)


def _read_views(scratch, M, D, Dkv, F):
    off = mq.chain_scratch_views(M, D, Dkv, F)
    raw = scratch.cpu().numpy()
    shapes = {"xn": (D, "bf16"), "qkv": (D + 2 * Dkv, "f32"), "a": (D, "bf16"), "o": (D, "f32"),
              "h1": (D, "f32"), "xn1": (D, "bf16"), "g": (F, "f32"), "u": (F, "f32"),
              "act": (F, "bf16"), "down": (D, "f32")}
    out = {}
    for name, (n, kind) in shapes.items():
        b = off[name]
        if kind == "f32":
            out[name] = raw[b:b + 4 * M * n].view(np.float32).reshape(M, n).astype(np.float64)
        else:
            out[name] = synth.f32_from_bf16_bits(raw[b:b + 2 * M * n].view(np.uint16).reshape(M, n)).astype(np.float64)
    return out


def check_layer_steps(v, ref, h_in, h_out, D, Dkv, hd, label):
    """Every step of one layer on the GPU's own inputs (see the module doc).
    h_in: the layer's input residual stream (fp32 values), or None when it is
    not known (a deeper layer): then the input norm and the first residual
    add are not checked."""
    def linear_ok(y, x, w, name):
        return check_linear(y, x, w, f"{label}: {name}")
    worst = 0.0
    if h_in is not None:
        v0 = och.rmsnorm(h_in)
        assert np.all(np.abs(v["xn"] - och.to_bf16(v0)) <= och.bf16_flip(v0, och.rmsnorm_f32_error(h_in))), label
    worst = max(worst, linear_ok(v["qkv"], v["xn"], ref["qkv"], "qkv"))
    assert np.array_equal(v["a"], och.to_bf16(och.attention_single_token(v["qkv"], D, Dkv, hd))), label
    worst = max(worst, linear_ok(v["o"], v["a"], ref["o"], "o"))
    if h_in is not None:
        assert np.array_equal(v["h1"], (h_in.astype(np.float32) + v["o"].astype(np.float32)).astype(np.float64)), label
    v1 = och.rmsnorm(v["h1"])
    assert np.all(np.abs(v["xn1"] - och.to_bf16(v1)) <= och.bf16_flip(v1, och.rmsnorm_f32_error(v["h1"]))), label
    worst = max(worst, linear_ok(v["g"], v["xn1"], ref["gate"], "gate"))
    worst = max(worst, linear_ok(v["u"], v["xn1"], ref["up"], "up"))
    pre = och.silu(v["g"]) * v["u"]
    assert np.all(np.abs(v["act"] - och.to_bf16(pre)) <= och.bf16_flip(pre, och.swiglu_f32_error(v["g"], v["u"]))), label
    worst = max(worst, linear_ok(v["down"], v["act"], ref["down"], "down"))
    assert np.array_equal(h_out, (v["h1"].astype(np.float32) + v["down"].astype(np.float32)).astype(np.float64)), label
    return worst


def sanity(h_gpu, h_ref, label, rel=1e-2):
    assert np.all(np.isfinite(h_gpu)), label
    dev = np.sqrt(np.mean((h_gpu - h_ref) ** 2)) / np.sqrt(np.mean(h_ref ** 2))
    assert dev <= rel, f"{label}: relative RMS deviation {dev:.3g}"
    return dev


@pytest.mark.parametrize("M", [1, 3])
def test_chain_small_every_depth(M):
    D, Dkv, F, hd = 512, 128, 1024, 64
    widths = [8, 4, 2, 3, 6]
    ref_layers, dev_layers, _keep = build_chain(5, widths, D, Dkv, F, 100)
    h0 = np.random.default_rng(M).standard_normal((M, D)).astype(np.float32).astype(np.float64)
    trace = []
    och.chain_forward(h0, ref_layers, D, Dkv, hd, trace=trace)
    for depth in range(1, 6):
        h, v = run_gpu(dev_layers[:depth], h0, M, D, Dkv, F, hd, views=True)
        w = check_layer_steps(v, ref_layers[depth - 1], h0 if depth == 1 else None, h, D, Dkv, hd,
                              f"depth {depth} M={M}")
        dev = sanity(h, trace[depth - 1], f"depth {depth} M={M}")
        print(f"depth {depth} M={M}: worst linear err/tol {w:.3f}, end-to-end relative RMS {dev:.2e}")


def test_chain_7b_shapes_two_layers():
    D, Dkv, F, hd, M = 4096, 1024, 14336, 128, 1
    ref_layers, dev_layers, _keep = build_chain(2, [8, 2], D, Dkv, F, 200)
    h0 = np.random.default_rng(7).standard_normal((M, D)).astype(np.float32).astype(np.float64)
    h_ref = och.chain_forward(h0, ref_layers, D, Dkv, hd)
    h1, v1 = run_gpu(dev_layers[:1], h0, M, D, Dkv, F, hd, views=True)
    check_layer_steps(v1, ref_layers[0], h0, h1, D, Dkv, hd, "7B layer 0")
    h, v = run_gpu(dev_layers, h0, M, D, Dkv, F, hd, views=True)
    w = check_layer_steps(v, ref_layers[1], None, h, D, Dkv, hd, "7B layer 1")
    print(f"7B shapes: worst linear err/tol {w:.3f}, end-to-end relative RMS {sanity(h, h_ref, '7B shapes'):.2e}")


def test_chain_graph_replay_matches_direct():
    # first call direct, second captured and launched, third replayed: every
    # call's last layer passes the step checks, and the calls agree with each
    # other to rounding
    D, Dkv, F, hd, M = 512, 128, 1024, 64, 2
    ref_layers, dev_layers, _keep = build_chain(3, [4, 2, 8], D, Dkv, F, 300)
    h0 = np.random.default_rng(9).standard_normal((M, D)).astype(np.float32).astype(np.float64)
    h_ref = och.chain_forward(h0, ref_layers, D, Dkv, hd)
    plan = mq.ChainPlan(dev_layers, M, D, Dkv, F, hd)
    scratch = torch.empty(mq.chain_scratch_bytes(M, D, Dkv, F), dtype=torch.uint8, device=DEV)
    h = torch.empty((M, D), dtype=torch.float32, device=DEV)
    s = torch.cuda.Stream()
    outs = []
    for i in range(4):
        with torch.cuda.stream(s):
            h.copy_(torch.from_numpy(h0.astype(np.float32)))
            plan.run(h, scratch, graph=True, stream=s)
        s.synchronize()
        mq.device_status(s)
        outs.append(h.cpu().numpy().astype(np.float64))
        check_layer_steps(_read_views(scratch, M, D, Dkv, F), ref_layers[2], None, outs[-1], D, Dkv, hd,
                          f"call {i}")
        sanity(outs[-1], h_ref, f"call {i}")
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
