"""The debug build (libmq_debug.so, compiled with MQ_DEBUG_BOUNDS): its device
index checks leave correct calls correct and turn a bad index into the
MQ_ERR_BOUNDS status instead of an out-of-range access.

The checks run in a child process that loads the debug library
(MQ_LIBRARY=debug); the bad index is an Extra Precision column past K, which
only that library is ever given (the child asserts it loaded the debug
build before making the call)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import os, sys
sys.path.insert(0, os.path.join(ROOT, "tests"))
sys.path.insert(0, ROOT)
import numpy as np
import torch
import nested_bit_weight_int8_b200 as mq
assert mq.LIB_PATH.endswith("libmq_debug.so"), mq.LIB_PATH
import oracle, synth
from gpu_util import DEV, check_linear, gpu_pack, to_dev, weights

n, k, m = 1000, 1024, 3
_, w = weights("gauss", n, k, 5)
q, a, z = oracle.quantize_minmax(w)
xb = synth.activations(m, k, 6)
xv = synth.f32_from_bf16_bits(xb).astype(np.float64)
qd, ad, zd, xd = to_dev(q), to_dev(a), to_dev(z), to_dev(xb)

# correct calls: planes, container, Extra Precision, prefill; status OK
for r in (8, 4, 2):
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
    mq.linear(xd, m, k, gpu_pack(qd, r), ad, zd, n, r, y)
    mq.device_status()
    check_linear(y.cpu().numpy().astype(np.float64), xv, oracle.dequant_slice(q, a, z, r), f"debug r={r}")
y = torch.full((m, n), float("nan"), dtype=torch.float32, device=DEV)
mq.linear_container(xd, m, k, qd, ad, zd, n, 4, True, y)
mq.device_status()
check_linear(y.cpu().numpy().astype(np.float64), xv, oracle.dequant_slice(q, a, z, 4), "debug container")
rows = torch.empty(n + 1, dtype=torch.int32, device=DEV)
mq.ep_overflow_rows(qd, n, k, 2, rows)
nnz = int(rows[n].item())
cols = torch.empty(max(nnz, 8), dtype=torch.int16, device=DEV)
mq.ep_overflow_cols(qd, n, k, 2, rows, cols)
p2 = gpu_pack(qd, 2)
mq.linear_ep(xd, m, k, p2, ad, zd, n, 2, rows, cols, y)
mq.device_status()
check_linear(y.cpu().numpy().astype(np.float64), xv, oracle.dequant_slice(q, a, z, 2, clamp=False), "debug ep")
mp = 64
xp = synth.activations(mp, k, 7)
yp = torch.full((mp, n), float("nan"), dtype=torch.float32, device=DEV)
mq.linear(to_dev(xp), mp, k, gpu_pack(qd, 8), ad, zd, n, 8, yp)
mq.device_status()
check_linear(yp.cpu().numpy().astype(np.float64), synth.f32_from_bf16_bits(xp).astype(np.float64),
             oracle.dequant_slice(q, a, z, 8), "debug prefill")

# a column past K in the list: the check skips the read and reports it
assert nnz > 0
cols[0] = k + 5
mq.linear_ep(xd, m, k, p2, ad, zd, n, 2, rows, cols, y)
try:
    mq.device_status()
    raise SystemExit("no bounds error reported")
except mq.MQError as e:
    assert e.status == mq.MQ_ERR_BOUNDS, e
# the library stays usable and the flag is cleared
mq.linear(xd, m, k, p2, ad, zd, n, 2, y)
mq.device_status()
print("debug-bounds ok")
'''


def test_debug_build_checks_indices():
    env = dict(os.environ, MQ_LIBRARY="debug")
    code = "ROOT = %r\n" % ROOT + CHILD
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "debug-bounds ok" in r.stdout
