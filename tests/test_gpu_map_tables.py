"""The bounded cache of tensor-map tables behind mq_stack_forward.

A launch of more than 8 linears reads its plane maps from a device table, one
per distinct list of linears. The cache keeps at most 64 tables, evicting the
least recently used; a table served during a CUDA graph capture is pinned for
the graph's sake. These tests drive more distinct lists through the stack than
the cache holds and check every product against the float64 oracle, the bound
on the table count, and a captured graph replayed after the evictions.
"""
import numpy as np
import pytest
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import synth
from gpu_util import DEV, check_linear, gpu_pack, to_dev

pytestmark = pytest.mark.gpu

N_LIN = 12
WIDTHS = [8, 4, 2, 6, 3, 4, 8, 2, 4, 6, 2, 8]


@pytest.fixture(scope="module")
def linears():
    out = []
    for i in range(N_LIN):
        n, k = 64 + 16 * i, 256 + 128 * (i % 3)
        w = synth.f32_from_bf16_bits(synth.gaussian_weights(n, k, 1200 + i)).astype(np.float64)
        q, a, z = oracle.quantize_minmax(w)
        r = WIDTHS[i]
        x_bits = synth.activations(1, k, 1300 + i)
        out.append(dict(n=n, k=k, r=r, packed=gpu_pack(to_dev(q), r), a=to_dev(a), z=to_dev(z),
                        x=to_dev(x_bits), xv=synth.f32_from_bf16_bits(x_bits).astype(np.float64),
                        wr=oracle.dequant_slice(q, a, z, r)))
    return out


def _plan(lins, order, ys):
    descs = [(lins[i]["x"], lins[i]["packed"], lins[i]["a"], lins[i]["z"], ys[i], lins[i]["n"], lins[i]["k"])
             for i in order]
    # one layer per linear, so each keeps its own width
    return mq.StackPlan(descs, list(range(len(order))), [lins[i]["r"] for i in order], 1)


def _fresh_outputs(lins):
    return [torch.full((1, L["n"]), float("nan"), dtype=torch.float32, device=DEV) for L in lins]


def _check_all(lins, ys, order, label):
    for i in order:
        check_linear(ys[i].cpu().numpy().astype(np.float64), lins[i]["xv"], lins[i]["wr"], f"{label} linear {i}")


def _orders(count, seed):
    rng = np.random.default_rng(seed)
    return [list(rng.permutation(N_LIN)[: 9 + (j % 4)]) for j in range(count)]


def test_cache_stays_bounded_and_results_hold(linears):
    mq.release_workspace()
    assert mq.debug_map_table_count() == 0
    orders = _orders(80, 5)
    for j, order in enumerate(orders):
        ys = _fresh_outputs(linears)
        _plan(linears, order, ys).run()
        mq.device_status()
        assert mq.debug_map_table_count() <= 64
        if j % 8 == 0 or j >= 76:
            _check_all(linears, ys, order, f"list {j}")
    assert mq.debug_map_table_count() == 64
    # the first list was evicted long ago: it is rebuilt and still right
    ys = _fresh_outputs(linears)
    _plan(linears, orders[0], ys).run()
    mq.device_status()
    _check_all(linears, ys, orders[0], "first list again")
    mq.release_workspace()
    assert mq.debug_map_table_count() == 0


def test_captured_table_survives_eviction(linears):
    mq.release_workspace()
    side = torch.cuda.Stream()
    order = list(range(N_LIN))
    ys = _fresh_outputs(linears)
    plan = _plan(linears, order, ys)
    with torch.cuda.stream(side):
        plan.run(side)                      # builds the table and the stream's workspace
    side.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        plan.run(side)
    side.synchronize()
    # fill the cache past its bound with other lists, on the default stream
    for other in _orders(70, 6):
        ys2 = _fresh_outputs(linears)
        _plan(linears, other, ys2).run()
    mq.device_status()
    assert mq.debug_map_table_count() <= 64
    for y in ys:
        y.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    mq.device_status(side)
    _check_all(linears, ys, order, "graph replay after evictions")
    del g
    torch.cuda.synchronize()
    mq.release_workspace()


def test_new_list_during_capture_is_refused(linears):
    mq.release_workspace()
    side = torch.cuda.Stream()
    order = list(range(N_LIN))
    ys = _fresh_outputs(linears)
    warm = _plan(linears, order[:9], ys)
    with torch.cuda.stream(side):
        warm.run(side)                      # the stream's workspace exists before capture
    side.synchronize()
    new = _plan(linears, order[::-1], ys)   # a list never served
    g = torch.cuda.CUDAGraph()
    err = None
    with torch.cuda.graph(g, stream=side):
        try:
            new.run(side)
        except mq.MQError as e:
            err = e
    assert err is not None and err.status == mq.MQ_ERR_CUDA
    del g
    torch.cuda.synchronize()
    mq.release_workspace()
