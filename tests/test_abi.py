"""C-ABI checks that need no GPU: the library loads, exports every function
include/mq.h declares, computes sizes, and rejects bad arguments on the host
before touching CUDA."""
import ctypes
import os
import re

import pytest

import nested_bit_weight_int8_b200 as mq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "mq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for want in ["mq_quantize_int8", "mq_slice_pack", "mq_linear", "mq_stack_forward",
                 "mq_packed_bytes", "mq_last_error"]:
        assert want in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(mq.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(mq.EXPORTED) == set(_declared_functions())


def test_version():
    assert mq.version() > 0


@pytest.mark.parametrize("r", [8, 6, 4, 3, 2])
def test_packed_bytes(r):
    assert mq.packed_bytes(14336, 4096, r) == 14336 * 4096 * r // 8
    assert mq.packed_bytes(1, 32, r) == (4 * r if r in (8, 4) else 0)
    assert mq.packed_bytes(1, 128, r) == 16 * r


# the K unit of each width: every plane row a whole number of 16-byte units
K_UNIT = {8: 32, 4: 32, 6: 64, 2: 64, 3: 128}


@pytest.mark.parametrize("r", [8, 6, 4, 3, 2])
def test_k_unit_per_width(r):
    u = K_UNIT[r]
    F = FAKE
    for k in (u, 3 * u, 4096 + u):
        assert mq.packed_bytes(4, k, r) == 4 * k * r // 8
    for k in (u // 2, u + 16, 3 * u - 16, 4096 + u // 2):
        if k % K_UNIT[r] == 0:
            continue
        assert mq.packed_bytes(4, k, r) == 0, (r, k)
        assert mq.raw_status("mq_slice_pack", F, 4, k, r, F, None) == mq.MQ_ERR_INVALID_ARG, (r, k)
        assert mq.raw_status("mq_linear", F, 1, k, F, F, F, 64, r, F, None) == mq.MQ_ERR_INVALID_ARG, (r, k)
        assert f"multiple of {u}" in mq.last_error()
    # the int8 container serves every width from K % 32
    assert mq.raw_status("mq_linear_container", F, 1, 80, F, F, F, 64, r, 1, F, None) == mq.MQ_ERR_INVALID_ARG
    assert "multiple of 32" in mq.last_error()


def test_packed_bytes_rejects():
    assert mq.packed_bytes(4, 48, 4) == 0      # K % 32
    assert mq.packed_bytes(4, 64, 5) == 0      # r
    assert mq.packed_bytes(0, 64, 4) == 0
    assert mq.packed_bytes(4, 0, 4) == 0


FAKE = 1 << 20  # an aligned non-null address; never dereferenced by rejected calls


@pytest.mark.parametrize("args,what", [
    ((FAKE, 1, 64, 256, FAKE, FAKE, FAKE, 4, FAKE, None), "ok-shape-bad-r"),
])
def test_linear_rejects_bad_width(args, what):
    x, M, K, p, a, z, N, r, y, s = args
    for bad_r in [0, 1, 5, 7, 9, 16]:
        st = mq.raw_status("mq_linear", x, M, K, p, a, z, N, bad_r, y, s)
        assert st == mq.MQ_ERR_INVALID_ARG
        assert "r=" in mq.last_error()


def test_linear_rejects_bad_shapes_and_pointers():
    F = FAKE
    cases = [
        (F, 0, 256, F, F, F, 64, 4, F),      # M = 0
        (F, 1, 80, F, F, F, 64, 4, F),       # K % 32 at r = 4
        (F, 1, 96, F, F, F, 64, 2, F),       # K % 64 at r = 2
        (F, 1, 192, F, F, F, 64, 3, F),      # K % 128 at r = 3
        (F, 1, 0, F, F, F, 64, 4, F),        # K = 0
        (F, 1, 256, F, F, F, 0, 4, F),       # N = 0
        (None, 1, 256, F, F, F, 64, 4, F),   # null x
        (F, 1, 256, None, F, F, 64, 4, F),   # null packed
        (F + 8, 1, 256, F, F, F, 64, 4, F),  # misaligned x
        (F, 1, 256, F + 4, F, F, 64, 4, F),  # misaligned packed
        (F, 1, 256, F, F + 2, F, 64, 4, F),  # misaligned alpha
    ]
    for c in cases:
        assert mq.raw_status("mq_linear", *c, None) == mq.MQ_ERR_INVALID_ARG, c
        assert mq.last_error()


def test_slice_pack_rejects():
    F = FAKE
    assert mq.raw_status("mq_slice_pack", F, 4, 48, 4, F, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_slice_pack", F, 4, 64, 5, F, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_slice_pack", None, 4, 64, 4, F, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_slice_pack", F + 1, 4, 64, 4, F, None) == mq.MQ_ERR_INVALID_ARG


def test_quantize_rejects():
    F = FAKE
    assert mq.raw_status("mq_quantize_int8", F, 7, 4, 64, F, F, F, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_quantize_int8", F, 1, 0, 64, F, F, F, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_quantize_int8", None, 1, 4, 64, F, F, F, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_quantize_int8", F + 2, 0, 4, 64, F, F, F, None) == mq.MQ_ERR_INVALID_ARG


def test_stack_rejects_bad_layers():
    F = FAKE
    lins = [(F, F, F, F, F, 64, 256)]
    with pytest.raises(mq.MQError) as e:
        mq.stack_forward(lins, [3], [4, 4], 1)
    assert e.value.status == mq.MQ_ERR_INVALID_ARG
    with pytest.raises(mq.MQError):
        mq.stack_forward(lins, [0], [5], 1)        # width 5
    with pytest.raises(mq.MQError):
        mq.stack_forward(lins, [0], [4], 33)       # M > 32


def test_linear_container_rejects():
    F = FAKE
    bad = [
        ((F, 1, 256, F, F, F, 64, 5, 1, F), mq.MQ_ERR_INVALID_ARG),    # r
        ((F, 1, 256, F, F, F, 64, 4, 2, F), mq.MQ_ERR_INVALID_ARG),    # clamp not 0/1
        ((F, 1, 80, F, F, F, 64, 4, 1, F), mq.MQ_ERR_INVALID_ARG),     # K % 32
        ((F, 1, 256, F + 4, F, F, 64, 4, 1, F), mq.MQ_ERR_INVALID_ARG),  # misaligned q
        ((F, 1, 256, None, F, F, 64, 4, 0, F), mq.MQ_ERR_INVALID_ARG),   # null q
    ]
    for c, want in bad:
        assert mq.raw_status("mq_linear_container", *c, None) == want, c
        assert mq.last_error()


def test_ep_entry_points_reject():
    F = FAKE
    assert mq.raw_status("mq_ep_overflow_rows", F, 4, 64, 8, F, None) == mq.MQ_ERR_INVALID_ARG  # r = 8
    assert mq.raw_status("mq_ep_overflow_rows", F, 4, 40, 2, F, None) == mq.MQ_ERR_INVALID_ARG  # K % 16
    assert mq.raw_status("mq_ep_overflow_rows", F + 8, 4, 64, 2, F, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_ep_overflow_rows", F, 4, 65552, 2, F, None) == mq.MQ_ERR_UNSUPPORTED
    assert mq.raw_status("mq_ep_overflow_cols", F, 4, 64, 2, F, None, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_ep_overflow_cols", F, 4, 64, 2, F + 2, F, None) == mq.MQ_ERR_INVALID_ARG
    ok = (F, 1, 256, F, F, F, 64)
    assert mq.raw_status("mq_linear_ep", *ok, 8, F, F, F, None) == mq.MQ_ERR_INVALID_ARG   # r = 8
    assert mq.raw_status("mq_linear_ep", *ok, 2, None, F, F, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_linear_ep", *ok, 2, F, F + 1, F, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_linear_ep", F, 1, 65600, F, F, F, 64, 2, F, F, F, None) == mq.MQ_ERR_UNSUPPORTED


def test_debug_build_exports_the_same_entry_points():
    # the build with device index checks (libmq_debug.so) is a drop-in
    # replacement: same header, same exported names
    import ctypes
    import os
    path = os.path.join(os.path.dirname(mq.LIB_PATH), "libmq_debug.so")
    if not os.path.exists(path):
        pytest.skip("libmq_debug.so not built")
    lib = ctypes.CDLL(path)
    for name in mq.EXPORTED:
        assert hasattr(lib, name), name


def test_quantize_clipped_rejects():
    F = FAKE
    ok = (F, 1, 4, 64)
    assert mq.raw_status("mq_quantize_int8_clipped", *ok, None, F, F, F, F, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_quantize_int8_clipped", *ok, F, None, F, F, F, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_quantize_int8_clipped", *ok, F + 2, F, F, F, F, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_quantize_int8_clipped", F, 7, 4, 64, F, F, F, F, F, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_quantize_int8_clipped", F, 1, 0, 64, F, F, F, F, F, None) == mq.MQ_ERR_INVALID_ARG


def test_chain_rejects_on_the_host():
    # every argument error is caught before anything launches (no GPU needed)
    import ctypes
    F = FAKE
    layer = mq.ChainLayer()
    layer.r = 4
    for i in range(5):
        layer.packed[i] = F
        layer.alpha[i] = F
        layer.zero[i] = F
    arr = (mq.ChainLayer * 1)(layer)
    need = mq.chain_scratch_bytes(1, 512, 128, 1024)
    assert need > 0
    base = (arr, 1, 1, 512, 128, 1024, 64, F, F, need, 0, None)

    def call(**kw):
        a = list(base)
        names = ["layers", "n", "M", "D", "Dkv", "F", "hd", "h", "scratch", "bytes", "flags", "stream"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return mq._chain(*a)

    assert call(n=0) == mq.MQ_ERR_INVALID_ARG
    assert call(M=0) == mq.MQ_ERR_INVALID_ARG
    assert call(M=33) == mq.MQ_ERR_INVALID_ARG
    assert call(D=500) == mq.MQ_ERR_INVALID_ARG
    assert call(hd=48) == mq.MQ_ERR_INVALID_ARG           # does not divide Dkv
    assert call(bytes=need - 1) == mq.MQ_ERR_INVALID_ARG
    assert call(scratch=F + 128) == mq.MQ_ERR_INVALID_ARG  # not 256-byte aligned
    assert call(flags=4) == mq.MQ_ERR_INVALID_ARG
    assert call(h=None) == mq.MQ_ERR_INVALID_ARG
    layer_bad = (mq.ChainLayer * 1)(layer)
    layer_bad[0].r = 5
    assert call(layers=layer_bad) == mq.MQ_ERR_INVALID_ARG
    assert mq.last_error()


def test_header_is_plain_c_and_links_from_c(tmp_path):
    # the boundary is a C ABI: the header compiles as C99 and a C program
    # links against the library and calls it (host-only calls, no GPU)
    import os
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(mq.LIB_PATH)
    src = tmp_path / "t.c"
    src.write_text(
        '#include "mq.h"\n'
        "int main(void) {\n"
        "  int64_t n = 0, k = 0;\n"
        '  if (mq_container_info("/nonexistent/x.mqc", &n, &k) != MQ_ERR_IO) return 1;\n'
        "  if (mq_packed_bytes(4, 64, 2) != 64) return 2;\n"
        "  return mq_version() > 0 ? 0 : 3;\n"
        "}\n")
    exe = tmp_path / "t"
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(root, "include"), str(src),
                        "-L", libdir, "-l:" + os.path.basename(mq.LIB_PATH), "-Wl,-rpath," + libdir,
                        "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert subprocess.run([str(exe)]).returncode == 0


def test_map_table_count_needs_no_device():
    # a host-side count of the tensor-map tables: none before any stack launch
    assert mq.debug_map_table_count() == 0
