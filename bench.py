"""Benchmark of the nested-bit int8 serving path on B200.

Headline workload: the Mix'n'Match 7B-shaped decode stack -- 32 layers x
(qkv 6144x4096, o 4096x4096, gate 14336x4096, up 14336x4096,
down 4096x14336), widths int8 on the first/last 4 layers, int4 on the next
4 inward, int2 on layers 8..23 -- streamed once per token (M = 1) through
mq_stack_forward. One step = one forward of every linear of the stack.
Metric: sliced-int GEMV effective HBM GB/s (packed-weight bytes / step
time), with % of the measured HBM peak and us/layer at r = 8, 4, 2.

The other parts of the path (int8 container quantize, slice-pack, a single
decode linear, the prefill GEMM) are timed separately and reported under
"rows".

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--M 1]
       python bench.py --impl reference ...   (CPU oracle arm)
For N > 1 launch under torch.distributed.run: every rank serves its own
replica of the stack (no data-path collective), value = sum over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np

import synth

WORKLOAD = "mixnmatch_7b_stack"
METRIC = "sliced-int GEMV effective HBM GB/s (% of peak) and us/layer at r=8/4/2"
L2_BYTES = 126 * 1024 * 1024


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1606.7)), "measured"
    return 6650.0, 1590.0, "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        import tempfile
        self.path = tempfile.mktemp(prefix="mq_clocks_", suffix=".csv")
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.fh, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)  # let the sampler start before the timed region
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        with open(self.path) as f:
            self.lines = [ln.strip() for ln in f]
        os.unlink(self.path)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------- distributed
def dist_setup(n_gpus: int):
    """Returns (rank, world, local_rank). Uses torch.distributed when launched
    by torch.distributed.run (WORLD_SIZE > 1)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def dist_max(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def dist_done(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------- GPU arm
class Stack:
    """The packed 7B Mix'n'Match stack resident in HBM."""

    def __init__(self, M: int, dev, layers: int = 32, seed_base: int = 1000, widths=None):
        import torch
        import nested_bit_weight_int8_b200 as mq
        self.mq, self.torch, self.dev, self.M = mq, torch, dev, M
        self.widths = list(widths) if widths else synth.mixnmatch_widths(layers)
        layers = len(self.widths)
        mats = synth.WORKLOADS[WORKLOAD]["mats"]
        self.Ks = sorted({k for _, _, k in mats})
        self.x = {k: synth.device_activations(M, k, 2000 + M + k, dev) for k in self.Ks}
        self.seed_base = seed_base
        self.lins, self.lol, self.bytes_by_width, self.layer_of = [], [], {}, []
        self.packed_bytes = 0
        self.rows_total = 0
        # all outputs live in one buffer so the result leaves the device in one copy
        n_out = sum(n for _, n, _ in mats) * layers
        self.y_all = torch.empty(M * n_out, dtype=torch.float32, device=dev)
        y_off = 0
        for layer in range(layers):
            r = self.widths[layer]
            for j, (_, n, k) in enumerate(mats):
                w = synth.device_gaussian_weights(n, k, seed_base + 5 * layer + j, dev)
                q = torch.empty((n, k), dtype=torch.uint8, device=dev)
                a = torch.empty(n, dtype=torch.float32, device=dev)
                z = torch.empty(n, dtype=torch.float32, device=dev)
                cur = torch.cuda.current_stream(dev)
                mq.quantize_int8(w, mq.MQ_BF16, n, k, q, a, z, cur)
                p = torch.empty(mq.packed_bytes(n, k, r), dtype=torch.uint8, device=dev)
                mq.slice_pack(q, n, k, r, p, cur)
                del w, q
                y = self.y_all[y_off:y_off + M * n].view(M, n)
                y_off += M * n
                self.lins.append((self.x[k], p, a, z, y, n, k))
                self.lol.append(layer)
                nb = n * k * r // 8
                self.packed_bytes += nb
                self.bytes_by_width[r] = self.bytes_by_width.get(r, 0) + nb
                self.rows_total += n
        self.layers = layers
        torch.cuda.synchronize()

    def step(self, stream=None):
        if getattr(self, "_plan", None) is None:
            self._plan = self.mq.StackPlan(self.lins, self.lol, self.widths, self.M)
        self._plan.run(stream)

    def sub_stack(self, width: int):
        """The linears of the layers at one width, as their own stack."""
        idx = [i for i, l in enumerate(self.lol) if self.widths[l] == width]
        layers = sorted({self.lol[i] for i in idx})
        remap = {l: j for j, l in enumerate(layers)}
        lins = [self.lins[i] for i in idx]
        lol = [remap[self.lol[i]] for i in idx]
        return lins, lol, [width] * len(layers), len(layers)

    def with_batch(self, M: int):
        """The stack's packed weights with inputs and outputs for batch M (the
        weights are not rebuilt): (lins, y buffer)."""
        import torch
        xs = {k: synth.device_activations(M, k, 2000 + M + k, self.dev) for k in self.Ks}
        n_out = sum(n for (_, _, _, _, _, n, _) in self.lins)
        y_all = torch.empty(M * n_out, dtype=torch.float32, device=self.dev)
        out, off = [], 0
        for (_, p, a, z, _, n, k) in self.lins:
            out.append((xs[k], p, a, z, y_all[off:off + M * n].view(M, n), n, k))
            off += M * n
        return out, y_all

    def lins_with_y(self, y_all):
        """The stack's linears with their outputs in another buffer of y_all's shape."""
        out, off = [], 0
        for (x, p, a, z, _, n, k) in self.lins:
            out.append((x, p, a, z, y_all[off:off + self.M * n].view(self.M, n), n, k))
            off += self.M * n
        return out

    def algorithmic_bytes(self) -> int:
        """Bytes the step must move: packed planes + alpha, z + x + y."""
        xb = sum(2 * self.M * k for (_, _, _, _, _, n, k) in self.lins)
        yb = sum(4 * self.M * n for (_, _, _, _, _, n, k) in self.lins)
        return self.packed_bytes + 8 * self.rows_total + xb + yb


def time_device(fn, steps: int, warmup: int, stream, world: int, dev, finish=None):
    """CUDA-event time of `steps` calls of fn on `stream`, barrier and
    synchronize on both sides, max over ranks. Returns ms per step.
    `finish`, if given, runs after the last call and before the end event
    (to join work the calls left on other streams into `stream`)."""
    import torch
    for _ in range(warmup):
        fn()
    if finish is not None:
        finish()
    torch.cuda.synchronize()
    dist_barrier(world, dev)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    if finish is not None:
        finish()
    e1.record(stream)
    torch.cuda.synchronize()
    dist_barrier(world, dev)
    ms = e0.elapsed_time(e1) / steps
    return dist_max(ms, world, dev)


def rows_timings(dev, stream):
    """Separately timed rows of the path on one 14336x4096 bf16 weight:
    quantize (Eq. 1 and Eq. 3's clipped variant), slice-pack (Eq. 6) per
    width, one decode linear per width (M = 1), the decode linear sliced on
    load from the container (Eq. 6 and Eq. 8), Extra Precision from the r = 2
    planes plus its sparse list, and the prefill GEMM at M = 2048 (from the
    planes, from the container, and with Extra Precision)."""
    import torch
    import nested_bit_weight_int8_b200 as mq
    n, k = 14336, 4096
    gen = torch.Generator(device=dev)
    gen.manual_seed(300)
    w = (torch.randn((n, k), generator=gen, device=dev) * 0.02).to(torch.bfloat16)
    q = torch.empty((n, k), dtype=torch.uint8, device=dev)
    a = torch.empty(n, dtype=torch.float32, device=dev)
    z = torch.empty(n, dtype=torch.float32, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def timed(fn, reps=10):
        fn()
        torch.cuda.synchronize()
        tot = 0.0
        for _ in range(reps):
            flush.zero_()
            # keep the GPU busy while the host enqueues the call, so that the
            # events bracket device time only, not the host's launch latency
            torch.cuda._sleep(200000)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            tot += e0.elapsed_time(e1)
        return tot / reps * 1000.0  # us

    out = {}
    us = timed(lambda: mq.quantize_int8(w, mq.MQ_BF16, n, k, q, a, z, stream))
    out["quantize_int8_14336x4096"] = {"us": round(us, 2), "GBps": round((n * k * 3 + 8 * n) / us / 1e3, 1)}
    # Eq. 3 clipped variant, per-row gamma, beta in [0.6, 1]
    gam = 0.6 + 0.4 * torch.rand(n, generator=gen, device=dev)
    bet = 0.6 + 0.4 * torch.rand(n, generator=gen, device=dev)
    qc = torch.empty_like(q)
    us = timed(lambda: mq.quantize_int8_clipped(w, mq.MQ_BF16, n, k, gam, bet, qc, a, z, stream))
    out["quantize_int8_clipped_14336x4096"] = {"us": round(us, 2),
                                               "GBps": round((n * k * 3 + 16 * n) / us / 1e3, 1)}
    mq.quantize_int8(w, mq.MQ_BF16, n, k, q, a, z, stream)
    del qc
    x = torch.randn((1, k), generator=gen, device=dev).to(torch.bfloat16)
    y = torch.empty((1, n), dtype=torch.float32, device=dev)
    for r in (8, 4, 2):
        p = torch.empty(mq.packed_bytes(n, k, r), dtype=torch.uint8, device=dev)
        us = timed(lambda: mq.slice_pack(q, n, k, r, p, stream))
        out[f"slice_pack_r{r}"] = {"us": round(us, 2), "GBps": round((n * k + n * k * r // 8) / us / 1e3, 1)}
        us = timed(lambda: mq.linear(x, 1, k, p, a, z, n, r, y, stream))
        out[f"decode_linear_r{r}_M1"] = {"us": round(us, 2), "GBps": round(n * k * r / 8 / us / 1e3, 1)}
    # Extra Precision (Eq. 8) from the r = 2 planes plus the sparse list of
    # extra-bucket positions, on weights with about 2.5% of each row there
    we = torch.randn((n, k), generator=gen, device=dev).clamp_(-4.0, 4.0)
    top = torch.rand((n, k), generator=gen, device=dev) < 0.025
    we = torch.where(top, 3.2 + 0.8 * torch.rand((n, k), generator=gen, device=dev), we)
    we[:, 0] = -4.0
    we[:, 1] = 4.0
    we = (we * 0.02).to(torch.bfloat16)
    qe = torch.empty_like(q)
    ae, ze = torch.empty_like(a), torch.empty_like(z)
    mq.quantize_int8(we, mq.MQ_BF16, n, k, qe, ae, ze, stream)
    del we, top
    pe = torch.empty(mq.packed_bytes(n, k, 2), dtype=torch.uint8, device=dev)
    mq.slice_pack(qe, n, k, 2, pe, stream)
    rows_e = torch.empty(n + 1, dtype=torch.int32, device=dev)
    mq.ep_overflow_rows(qe, n, k, 2, rows_e, stream)
    torch.cuda.synchronize()
    nnz = int(rows_e[n].item())
    cols_e = torch.empty(max(nnz, 8), dtype=torch.int16, device=dev)
    mq.ep_overflow_cols(qe, n, k, 2, rows_e, cols_e, stream)
    us = timed(lambda: mq.linear_ep(x, 1, k, pe, ae, ze, n, 2, rows_e, cols_e, y, stream))
    ep_bytes = n * k * 2 // 8 + 2 * nnz + 4 * (n + 1)
    out["decode_linear_ep_r2_M1"] = {"us": round(us, 2), "GBps": round(ep_bytes / us / 1e3, 1),
                                     "extra_bucket_frac": round(nnz / (n * k), 4),
                                     "bits_per_weight": round(8 * ep_bytes / (n * k), 3)}
    us = timed(lambda: mq.linear(x, 1, k, pe, ae, ze, n, 2, y, stream))
    out["decode_linear_eq6_same_planes_r2_M1"] = {"us": round(us, 2)}
    del qe, pe, rows_e, cols_e
    # slice on load from the int8 container (8 bits per weight streamed)
    for r in (4, 2):
        for clamp, tag in ((True, "eq6"), (False, "eq8")):
            us = timed(lambda: mq.linear_container(x, 1, k, q, a, z, n, r, clamp, y, stream))
            out[f"decode_container_r{r}_{tag}_M1"] = {"us": round(us, 2), "GBps": round(n * k / us / 1e3, 1)}
    # prefill GEMM on the 9B-shaped matrices, M = 2048, the interpolative widths
    bf16_peak = _peaks()[1]
    m = 2048
    for name, n_p, k_p, seed in (("up", 14336, 3584, 500), ("down", 3584, 14336, 501)):
        gen.manual_seed(seed)
        w_p = (torch.randn((n_p, k_p), generator=gen, device=dev) * 0.02).to(torch.bfloat16)
        q_p = torch.empty((n_p, k_p), dtype=torch.uint8, device=dev)
        a_p = torch.empty(n_p, dtype=torch.float32, device=dev)
        z_p = torch.empty(n_p, dtype=torch.float32, device=dev)
        mq.quantize_int8(w_p, mq.MQ_BF16, n_p, k_p, q_p, a_p, z_p, stream)
        del w_p
        xm = torch.randn((m, k_p), generator=gen, device=dev).to(torch.bfloat16)
        ym = torch.empty((m, n_p), dtype=torch.float32, device=dev)
        for r in (6, 4, 3, 2):
            p_p = torch.empty(mq.packed_bytes(n_p, k_p, r), dtype=torch.uint8, device=dev)
            mq.slice_pack(q_p, n_p, k_p, r, p_p, stream)
            us = timed(lambda: mq.linear(xm, m, k_p, p_p, a_p, z_p, n_p, r, ym, stream), reps=5)
            tf = 2 * m * n_p * k_p / us / 1e6
            out[f"prefill_{name}_{n_p}x{k_p}_r{r}_M{m}"] = {
                "us": round(us, 2), "TFLOPs": round(tf, 1),
                "frac_of_bf16_peak": round(tf / bf16_peak, 3)}
            del p_p
        # the same product sliced on load from the container (Eq. 6 at r = 4, Eq. 8 at r = 2)
        for r, clamp, tag in ((4, True, "eq6"), (2, False, "eq8")):
            us = timed(lambda: mq.linear_container(xm, m, k_p, q_p, a_p, z_p, n_p, r, clamp, ym, stream),
                       reps=5)
            tf = 2 * m * n_p * k_p / us / 1e6
            out[f"prefill_container_{name}_r{r}_{tag}_M{m}"] = {
                "us": round(us, 2), "TFLOPs": round(tf, 1), "frac_of_bf16_peak": round(tf / bf16_peak, 3)}
        # Extra Precision (Eq. 8) at r = 2 from the planes plus the list of
        # extra-bucket positions (of these Gaussian weights, the top tail)
        p2 = torch.empty(mq.packed_bytes(n_p, k_p, 2), dtype=torch.uint8, device=dev)
        mq.slice_pack(q_p, n_p, k_p, 2, p2, stream)
        rows_p = torch.empty(n_p + 1, dtype=torch.int32, device=dev)
        mq.ep_overflow_rows(q_p, n_p, k_p, 2, rows_p, stream)
        torch.cuda.synchronize()
        nnz_p = int(rows_p[n_p].item())
        cols_p = torch.empty(max(nnz_p, 8), dtype=torch.int16, device=dev)
        mq.ep_overflow_cols(q_p, n_p, k_p, 2, rows_p, cols_p, stream)
        us = timed(lambda: mq.linear_ep(xm, m, k_p, p2, a_p, z_p, n_p, 2, rows_p, cols_p, ym, stream), reps=5)
        tf = 2 * m * n_p * k_p / us / 1e6
        out[f"prefill_linear_ep_{name}_r2_M{m}"] = {
            "us": round(us, 2), "TFLOPs": round(tf, 1), "frac_of_bf16_peak": round(tf / bf16_peak, 3),
            "extra_bucket_frac": round(nnz_p / (n_p * k_p), 5)}
        del q_p, xm, ym, p2, rows_p, cols_p
    torch.cuda.synchronize()
    return out


def configs_timings(dev, stream, stack, hbm_peak, steps):
    """The per-configuration decode numbers, each on its own shapes and laws:
    single linear (512 x 1024 fp32 weights, r = 8, 4, 2, M = 1); a Gemma-2-2B
    decode layer (q, k, v, o 2304 x 2304, gate, up 9216 x 2304, down
    2304 x 9216) at r = 4, M = 1, 4, 8, one grouped launch per layer; the
    Mistral-7B MLP (14336 x 4096 and 4096 x 14336, Student-t(4) * 0.02) at
    r = 2, 4, 8 and M = 1, 4, 16, 32, one launch per MLP; and the 7B
    Mix'n'Match stack at M = 2, 4, 8, 16, 32. The small configurations fit in
    L2, so each is timed round robin over enough copies of its weights
    (packed planes, alpha, z) to span at least 4x L2; every time is device time
    (CUDA events) per call, after warm-up."""
    import torch
    import nested_bit_weight_int8_b200 as mq
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", L2_BYTES)

    def quantized(w_dev, dtype_code, n, k):
        q = torch.empty((n, k), dtype=torch.uint8, device=dev)
        a = torch.empty(n, dtype=torch.float32, device=dev)
        z = torch.empty(n, dtype=torch.float32, device=dev)
        mq.quantize_int8(w_dev, dtype_code, n, k, q, a, z, stream)
        return q, a, z

    def copies(packed_bytes):
        return max(4, int(4 * l2 // max(1, packed_bytes)) + 1)

    def time_round_robin(plans, reps):
        """Device time per call of one pass over `plans`, replayed from a CUDA
        graph (launched directly, the host's enqueue rate would set the pace
        of such short calls)."""
        for _ in range(2):
            for pl in plans:
                pl.run(stream)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for pl in plans:
                pl.run(stream)
        graph.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        del graph
        return e0.elapsed_time(e1) * 1000.0 / (reps * len(plans))  # us per call

    def entry(us, packed, M):
        gbs = packed / (us * 1e-6) / 1e9
        return {"us": round(us, 2), "GBps": round(gbs, 1), "frac_of_hbm": round(gbs / hbm_peak, 3),
                "tokens_per_s": round(M / (us * 1e-6), 1)}

    out = {}
    # config 1: one 512 x 1024 linear, fp32 weights N(0, 0.02^2), seed 0
    n, k = 512, 1024
    w = torch.from_numpy(synth.gaussian_weights(n, k, 0, dtype="f32")).to(dev)
    q, a, z = quantized(w, mq.MQ_F32, n, k)
    x = torch.from_numpy(synth.activations(1, k, 1).view(np.int16)).to(dev)
    c1 = {}
    for r in (8, 4, 2):
        nb = n * k * r // 8
        lins = []
        for _ in range(copies(nb)):
            p = torch.empty(mq.packed_bytes(n, k, r), dtype=torch.uint8, device=dev)
            mq.slice_pack(q, n, k, r, p, stream)
            lins.append(mq.StackPlan([(x, p, a.clone(), z.clone(), torch.empty((1, n), dtype=torch.float32, device=dev), n, k)],
                                     [0], [r], 1))
        c1[f"r{r}_M1"] = entry(time_round_robin(lins, 3), nb, 1)
    out["single_linear_512x1024_f32"] = c1
    del w, q, lins
    # config 2: a Gemma-2-2B decode layer at r = 4, one grouped launch
    mats = synth.WORKLOADS["gemma2_2b_decode_layer"]["mats"]
    base = []
    for i, (_, n, k) in enumerate(mats):
        w = synth.device_gaussian_weights(n, k, 100 + i, dev)
        q, a, z = quantized(w, mq.MQ_BF16, n, k)
        p = torch.empty(mq.packed_bytes(n, k, 4), dtype=torch.uint8, device=dev)
        mq.slice_pack(q, n, k, 4, p, stream)
        base.append((p, a, z, n, k))
        del w, q
    layer_bytes = sum(n * k * 4 // 8 for (_, _, _, n, k) in base)
    c2 = {}
    n_copies = copies(layer_bytes)
    layers = [[(p.clone(), a.clone(), z.clone(), n, k) for (p, a, z, n, k) in base] for _ in range(n_copies)]
    for M in (1, 4, 8):
        xs = {k: synth.device_activations(M, k, 200 + M + k, dev) for k in {k for (*_, k) in base}}
        plans = []
        for lay in layers:
            lins = [(xs[k], p, a, z, torch.empty((M, n), dtype=torch.float32, device=dev), n, k)
                    for (p, a, z, n, k) in lay]
            plans.append(mq.StackPlan(lins, [0] * len(lins), [4], M))
        c2[f"r4_M{M}"] = entry(time_round_robin(plans, 3), layer_bytes, M)
    c2["per"] = "layer (7 linears, one launch)"
    out["gemma2_2b_layer_r4"] = c2
    del layers, base
    # config 3: the Mistral-7B MLP, heavy-tailed weights, r = 2, 4, 8
    mats = synth.WORKLOADS["mistral7b_mlp_heavy_tail"]["mats"]
    qs = []
    for i, (_, n, k) in enumerate(mats):
        w = torch.from_numpy(synth.student_t_weights(n, k, 300 + i).view(np.int16)).to(dev)
        qs.append((*quantized(w, mq.MQ_BF16, n, k), n, k))
        del w
    c3 = {}
    for r in (2, 4, 8):
        mlp_bytes = sum(n * k * r // 8 for (*_, n, k) in qs)
        n_copies = copies(mlp_bytes)
        packs = []
        for (q, a, z, n, k) in qs:
            p = torch.empty(mq.packed_bytes(n, k, r), dtype=torch.uint8, device=dev)
            mq.slice_pack(q, n, k, r, p, stream)
            packs.append((p, a, z, n, k))
        mlps = [[(p.clone(), a.clone(), z.clone(), n, k) for (p, a, z, n, k) in packs] for _ in range(n_copies)]
        for M in (1, 4, 16, 32):
            xs = {k: synth.device_activations(M, k, 400 + M + k, dev) for k in {k for (*_, k) in qs}}
            plans = [mq.StackPlan([(xs[k], p, a, z, torch.empty((M, n), dtype=torch.float32, device=dev), n, k)
                                   for (p, a, z, n, k) in mlp], [0, 0], [r], M) for mlp in mlps]
            c3[f"r{r}_M{M}"] = entry(time_round_robin(plans, 3), mlp_bytes, M)
        del mlps, packs
    c3["per"] = "MLP (up 14336x4096 + down 4096x14336, one launch)"
    out["mistral7b_mlp_student_t"] = c3
    del qs
    # config 4 at larger batches: the same packed stack, new inputs per M
    c4 = {}
    for M in (2, 4, 8, 16, 32):
        lins, y_all = stack.with_batch(M)
        plan = mq.StackPlan(lins, stack.lol, stack.widths, M)
        ms = time_device(lambda: plan.run(stream), max(3, steps // 8), 3, stream, 1, dev)
        c4[f"M{M}"] = entry(ms * 1000.0, stack.packed_bytes, M)
        c4[f"M{M}"]["us_per_layer"] = round(ms * 1000.0 / stack.layers, 2)
        del lins, y_all, plan
    c4["per"] = "step (32 layers, 160 linears, one launch)"
    out["mixnmatch_7b_stack_batches"] = c4
    torch.cuda.synchronize()
    return out


def cpu_baseline(M: int, budget_s: float = 12.0):
    """The CPU oracle (float64 numpy) on a bounded sample of the same
    workload: dequantize-and-multiply for row blocks of the stack's linears,
    repeated until about budget_s seconds of wall time (drawing each block's
    weights and quantizing them counts toward the wall time, not toward the
    timed oracle work). Returns the same metric (effective packed-weight GB/s)
    and what the sample was."""
    import oracle
    widths = synth.mixnmatch_widths(32)
    shapes = synth.stack_shapes(32)
    rows = 512
    done_bytes, t_used, n_blocks = 0, 0.0, 0
    picks = [0, 5 * 4 + 2, 5 * 12 + 4, 5 * 16 + 1, 5 * 31 + 3]  # linears at r = 8, 4, 2, 2, 8
    i = 0
    t_start = time.perf_counter()
    while (i == 0 or time.perf_counter() - t_start < budget_s) and i < 400:
        layer, name, n, k, seed = shapes[picks[i % len(picks)]]
        r = widths[layer]
        w = synth.f32_from_bf16_bits(synth.gaussian_weights(rows, k, seed + 7919 * i)).astype(np.float64)
        x = synth.f32_from_bf16_bits(synth.activations(M, k, 2000 + M + k)).astype(np.float64)
        q, a, z = oracle.quantize_minmax(w)
        t0 = time.perf_counter()
        y = oracle.linear(x, oracle.dequant_slice(q, a, z, r))
        t_used += time.perf_counter() - t0
        done_bytes += rows * k * r // 8
        n_blocks += 1
        i += 1
        del y
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count()
    return {"value": round(done_bytes / t_used / 1e9, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{n_blocks} blocks of {rows} rows from stack linears at their widths "
                      f"(dequantize + float64 matmul per block, M={M}), {t_used:.1f}s of CPU work"}


def run_gpu(args, rank, world, local):
    import torch
    import nested_bit_weight_int8_b200 as mq
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    hbm_peak, bf16_peak, peak_kind = _peaks()
    with torch.cuda.stream(stream):
        widths = [int(v) for v in args.widths.split(",")] if args.widths else None
        stack = Stack(args.M, dev, layers=args.layers, widths=widths)
        stack.step(stream)
        torch.cuda.synchronize()
        mq.device_status(stream)
        launches_per_step = 2 * ((len(stack.lins) + 255) // 256)

        clocks = ClockSampler(local)
        clocks.start()
        ms = time_device(lambda: stack.step(stream), args.steps, args.warmup, stream, world, dev)
        clk = clocks.stop()
        mq.device_status(stream)

        # us/layer at each width: the layers of one width as their own stack
        per_width = {}
        for r in sorted(set(stack.widths), reverse=True):
            lins, lol, wd, nl = stack.sub_stack(r)
            plan = mq.StackPlan(lins, lol, wd, args.M)
            msr = time_device(lambda: plan.run(stream),
                              max(3, args.steps // 4), 3, stream, world, dev)
            per_width[f"r{r}"] = {"layers": nl, "us_per_layer": round(msr * 1000 / nl, 2),
                                  "GBps": round(stack.bytes_by_width[r] / (msr * 1e-3) / 1e9, 1)}

        # Chained decode step (mq_chain_forward): each layer's output feeds the
        # next through the stand-in glue, so a token is a chain of dependent
        # launches; timed directly and replayed from a captured CUDA graph.
        chain = None
        if not args.no_chain and WORKLOAD == "mixnmatch_7b_stack" and len(stack.lins) == 5 * stack.layers:
            D, Dkv, F, hd = 4096, 1024, 14336, 128
            clayers = [(stack.widths[l], [(p, a, z) for (_, p, a, z, _, _, _) in stack.lins[5 * l:5 * l + 5]])
                       for l in range(stack.layers)]
            cplan = mq.ChainPlan(clayers, args.M, D, Dkv, F, hd)
            cscratch = torch.empty(mq.chain_scratch_bytes(args.M, D, Dkv, F), dtype=torch.uint8, device=dev)
            gen_h = torch.Generator(device=dev)
            gen_h.manual_seed(77)
            h_res = torch.randn((args.M, D), generator=gen_h, device=dev)
            n_chain = max(3, args.steps // 4)
            ms_direct = time_device(lambda: cplan.run(h_res, cscratch, False, stream), n_chain, 3, stream,
                                    world, dev)
            ms_graph = time_device(lambda: cplan.run(h_res, cscratch, True, stream), n_chain, 3, stream,
                                   world, dev)
            mq.device_status(stream)
            chain = {"layers": stack.layers, "launches_per_token": 1 + 12 * stack.layers,
                     "us_per_token_direct": round(ms_direct * 1000, 1),
                     "us_per_token_graph": round(ms_graph * 1000, 1),
                     "GBps_graph": round(stack.packed_bytes / (ms_graph * 1e-3) / 1e9, 1),
                     "glue": "RMSNorm, single-token attention, SwiGLU, fp32 residual (stand-in)"}
            del cscratch

        # End to end through the C ABI with host buffers: every step copies its
        # x in from pinned host memory and every output y back out. As a
        # serving loop would, it double-buffers y and copies step k's outputs
        # out on a second stream while step k + 1 computes.
        xs_host = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in stack.x.items()}
        for k, v in xs_host.items():
            v.copy_(stack.x[k].cpu())
        y_host = [torch.empty(stack.y_all.shape, dtype=torch.float32, pin_memory=True) for _ in range(2)]
        h2d = sum(v.numel() * v.element_size() for v in xs_host.values())
        d2h = y_host[0].numel() * 4
        y_dev = [stack.y_all, torch.empty_like(stack.y_all)]
        plans = [mq.StackPlan(stack.lins, stack.lol, stack.widths, args.M),
                 mq.StackPlan(stack.lins_with_y(y_dev[1]), stack.lol, stack.widths, args.M)]
        copy_stream = torch.cuda.Stream(device=dev)
        done = [torch.cuda.Event(), torch.cuda.Event()]   # step's outputs computed
        out_ok = [None, None]                             # step's outputs copied out
        k_step = [0]

        def e2e_step():
            b = k_step[0] % 2
            k_step[0] += 1
            if out_ok[b] is not None:
                stream.wait_event(out_ok[b])   # y buffer b is free again
            for k, v in xs_host.items():
                stack.x[k].copy_(v, non_blocking=True)
            plans[b].run(stream)
            done[b].record(stream)
            copy_stream.wait_event(done[b])
            with torch.cuda.stream(copy_stream):
                y_host[b].copy_(y_dev[b], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy_stream)
            out_ok[b] = ev

        def e2e_finish():
            stream.wait_stream(copy_stream)

        ms_e2e = time_device(e2e_step, max(3, args.steps // 4), 3, stream, world, dev, finish=e2e_finish)

        rows = rows_timings(dev, stream) if rank == 0 and not args.no_rows else {}
        configs = (configs_timings(dev, stream, stack, hbm_peak, args.steps)
                   if rank == 0 and not args.no_configs and WORKLOAD == "mixnmatch_7b_stack"
                   and len(stack.lins) == 160 and args.M == 1 else {})
    torch.cuda.synchronize()

    gbs = stack.packed_bytes / (ms * 1e-3) / 1e9
    algo = stack.algorithmic_bytes()
    achieved = algo / (ms * 1e-3) / 1e9
    # The driver keeps the tail of the printed line, so the long "rows" block
    # comes first and the per-width and per-configuration numbers last.
    out = {
        "rows": rows,
        "metric": METRIC,
        "value": round(gbs * world, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded torch normal weights N(0,0.02^2), activations N(0,1))",
        "config": {
            "workload": WORKLOAD,
            "layers": stack.layers,
            "widths": ("int8 x8 (layers 0-3, 28-31), int4 x8 (4-7, 24-27), int2 x16 (8-23)"
                       if stack.widths == synth.mixnmatch_widths(32) else stack.widths),
            "M": args.M,
            "linears": len(stack.lins),
            "packed_bytes_per_step": stack.packed_bytes,
            "arithmetic": "bf16 activations x exact integer codes (bf16), fp32 accumulate",
            "l2": "inputs larger than L2: 3.49 GB of packed planes streamed per step",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        },
        "pct_of_hbm_peak": round(100 * gbs / hbm_peak, 1),
        "us_per_layer": round(ms * 1000 / stack.layers, 2),
        "tokens_per_s": round(args.M * world * 1000.0 / ms, 1),
        "chain": chain,
        "roofline": {
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "peak": hbm_peak,
            "unit": "GB/s",
            "frac": round(achieved / hbm_peak, 4),
            "traffic": None,
            "peak_kind": peak_kind,
            "kernel": "gemv_streamk_kernel (timed with its prep kernel, one step)",
        },
        "e2e": {
            "value": round(stack.packed_bytes / (ms_e2e * 1e-3) / 1e9 * world, 1),
            "unit": "GB/s",
            "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "ms_per_step": round(ms_e2e, 4),
            "overlap": "y double-buffered; step k's outputs copied to pinned host memory on a second "
                       "stream while step k + 1 computes",
        },
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    tr = _profile_traffic()
    if tr is not None and tr.get("kernel_source_hash") == _kernel_hash():
        out["roofline"]["traffic"] = tr.get("dram_bytes_per_launch")
    out["configs"] = configs
    out["per_width"] = per_width
    return out


def _profile_traffic():
    """DRAM bytes per launch of the stack kernel from the committed ncu
    summary (lines "key: value"), or None."""
    path = os.path.join(ROOT, "profiles", "gemv_streamk_mixnmatch_7b_M1.md")
    if not os.path.exists(path):
        return None
    d = {}
    with open(path) as f:
        for ln in f:
            if ":" in ln and not ln.startswith("#"):
                k, v = ln.split(":", 1)
                d[k.strip().strip("-* `")] = v.strip().strip("`")
    try:
        return {"dram_bytes_per_launch": float(d["dram_bytes_per_launch"]),
                "kernel_source_hash": d["kernel_source_hash"]}
    except (KeyError, ValueError):
        return None


# The sources the stack's decode kernels (gemv_prep_kernel, gemv_streamk_kernel)
# are built from: their DRAM counters stay valid while these are unchanged.
KERNEL_SOURCES = ("gemv.cu", "mq_device.cuh", "mq_internal.h", "tensor_map.cu")


def _kernel_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "nested_bit_weight_int8_b200", "csrc")
    for name in KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def run_reference(args, rank, world):
    """CPU oracle arm: the float64 oracle on the host cores, each step a
    bounded sample of the same workload, same metric and unit."""
    budget = max(1.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(args.M, budget_s=budget / 4)
    vals, walls = [], []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        vals.append(cpu_baseline(args.M, budget_s=budget))
        walls.append(time.perf_counter() - t0)
    v = float(np.median([b["value"] for b in vals]))
    last = vals[-1]
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(v, 4),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        # wall time of one step, which is a bounded sample of the workload
        # (`config.sample`), not a whole pass over the stack
        "ms_per_step": round(1000.0 * float(np.mean(walls)), 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded numpy PCG64)",
        "config": {"workload": WORKLOAD, "M": args.M, "sample": last["sample"]},
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": last["cores"],
                         "kind": "oracle", "sample": last["sample"]},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def emit(line: dict, results: str = "") -> None:
    """Prints the JSON line; with --results, also appends it (with a UTC time
    stamp) to that JSON-lines file."""
    print(json.dumps(line), flush=True)
    if results:
        import datetime
        rec = dict(line, time_utc=datetime.datetime.now(datetime.timezone.utc).isoformat(timespec="seconds"))
        os.makedirs(os.path.dirname(os.path.abspath(results)), exist_ok=True)
        with open(results, "a") as f:
            f.write(json.dumps(rec) + "\n")


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--layers", type=int, default=32,
                    help="layers of the 7B-shaped stack (widths follow the Mix'n'Match pattern)")
    ap.add_argument("--widths", default="",
                    help="comma-separated per-layer widths; overrides --layers (small profiling stacks)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-rows", action="store_true")
    ap.add_argument("--no-chain", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration decode timings (configs 1-3, stack at M = 2..32)")
    ap.add_argument("--results", default="",
                    help="also append each JSON line, time-stamped, to this JSON-lines file")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--rows-only", action="store_true",
                    help="time only the separate rows (quantize, slice-pack, one decode linear, "
                         "prefill GEMMs) and print them; small enough for profiler captures")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        # the CPU oracle arm: rank 0 alone runs and prints; other ranks exit
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if int(os.environ.get("RANK", "0")) == 0:
            emit(run_reference(args, 0, world), args.results)
        return 0
    if args.rows_only:
        import torch
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        stream = torch.cuda.Stream(device=dev)
        with torch.cuda.stream(stream):
            rows = rows_timings(dev, stream)
        emit({"rows": rows}, args.results)
        return 0
    rank, world, local = dist_setup(args.gpus)
    try:
        out = run_gpu(args, rank, world, local)
        if rank == 0:
            if not args.no_cpu:
                # before the per-width and per-configuration blocks, which stay last
                cb = cpu_baseline(args.M)
                tail = {key: out.pop(key) for key in ("configs", "per_width")}
                out["cpu_baseline"] = cb
                out.update(tail)
            emit(out, args.results)
        return 0
    finally:
        dist_done(world)


if __name__ == "__main__":
    sys.exit(main())
