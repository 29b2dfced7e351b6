"""Python binding of libmq.so, the nested-bit int8 (Matryoshka Quantization)
serving path for B200.

Argument marshalling only: every function forwards to the C ABI declared in
include/mq.h, and every step of the path runs in the library's CUDA kernels.
There is no CPU fallback: importing this package fails if libmq.so is missing
or cannot be loaded.

Pointers are plain integers (device addresses unless documented otherwise);
helpers accept torch tensors for convenience and pass their data_ptr().
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# MQ_LIBRARY=debug loads the build with device index checks (libmq_debug.so).
LIB_PATH = os.path.join(_HERE, "libmq_debug.so" if os.environ.get("MQ_LIBRARY") == "debug"
                        else "libmq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python nested_bit_weight_int8_b200/build.py` "
        "(nvcc, sm_100a). There is no fallback implementation.")
_lib = ctypes.CDLL(LIB_PATH)

(MQ_OK, MQ_ERR_INVALID_ARG, MQ_ERR_UNSUPPORTED, MQ_ERR_CUDA, MQ_ERR_TIMEOUT, MQ_ERR_BOUNDS,
 MQ_ERR_IO) = range(7)
MQ_F32, MQ_BF16 = 0, 1
WIDTHS = (8, 6, 4, 3, 2)

_i64, _int, _vp, _u64 = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_uint64


class LinearDesc(ctypes.Structure):
    """mq_linear_desc: one linear of a Mix'n'Match stack."""
    _fields_ = [("x", _vp), ("packed", _vp), ("alpha", _vp), ("zero", _vp), ("y", _vp),
                ("N", _i64), ("K", _i64)]


class ChainLayer(ctypes.Structure):
    """mq_chain_layer: one layer of a chained stack (qkv, o, gate, up, down at width r)."""
    _fields_ = [("r", _int), ("packed", _vp * 5), ("alpha", _vp * 5), ("zero", _vp * 5)]


MQ_CHAIN_GRAPH = 1


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_version = _sig("mq_version", _int, [])
_last_error = _sig("mq_last_error", ctypes.c_char_p, [])
_packed_bytes = _sig("mq_packed_bytes", ctypes.c_size_t, [_i64, _i64, _int])
_quantize = _sig("mq_quantize_int8", _int, [_vp, _int, _i64, _i64, _vp, _vp, _vp, _vp])
_quantize_clipped = _sig("mq_quantize_int8_clipped", _int,
                        [_vp, _int, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp])
_slice_pack = _sig("mq_slice_pack", _int, [_vp, _i64, _i64, _int, _vp, _vp])
_linear = _sig("mq_linear", _int, [_vp, _i64, _i64, _vp, _vp, _vp, _i64, _int, _vp, _vp])
_stack = _sig("mq_stack_forward", _int,
              [ctypes.POINTER(LinearDesc), ctypes.POINTER(_int), _int, ctypes.POINTER(_int), _int,
               _i64, _vp])
_linear_container = _sig("mq_linear_container", _int,
                         [_vp, _i64, _i64, _vp, _vp, _vp, _i64, _int, _int, _vp, _vp])
_ovf_rows = _sig("mq_ep_overflow_rows", _int, [_vp, _i64, _i64, _int, _vp, _vp])
_ovf_cols = _sig("mq_ep_overflow_cols", _int, [_vp, _i64, _i64, _int, _vp, _vp, _vp])
_linear_ep = _sig("mq_linear_ep", _int,
                  [_vp, _i64, _i64, _vp, _vp, _vp, _i64, _int, _vp, _vp, _vp, _vp])
_chain_bytes = _sig("mq_chain_scratch_bytes", ctypes.c_size_t, [_i64, _i64, _i64, _i64])


class ChainViews(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("xn", "qkv", "a", "o", "h1", "xn1", "g", "u", "act", "down")]


_chain_views = _sig("mq_chain_scratch_views", _int, [_i64, _i64, _i64, _i64, ctypes.POINTER(ChainViews)])
_chain = _sig("mq_chain_forward", _int,
              [ctypes.POINTER(ChainLayer), _int, _i64, _i64, _i64, _i64, _i64, _vp, _vp,
               ctypes.c_size_t, _int, _vp])
_c_save = _sig("mq_container_save", _int, [ctypes.c_char_p, _vp, _vp, _vp, _i64, _i64])
_c_info = _sig("mq_container_info", _int,
               [ctypes.c_char_p, ctypes.POINTER(_i64), ctypes.POINTER(_i64)])
_c_load = _sig("mq_container_load", _int, [ctypes.c_char_p, _vp, _vp, _vp, _i64, _i64])
_linear_noalloc = _sig("mq_linear_noalloc", _int,
                      [_vp, _i64, _i64, _vp, _vp, _vp, _i64, _int, _vp, _vp])
_device_status = _sig("mq_device_status", _int, [_vp])
_release = _sig("mq_release_workspace", _int, [])
_wait_limit = _sig("mq_debug_set_wait_limit_ns", _int, [_u64])
_map_count = _sig("mq_debug_map_table_count", _i64, [])

EXPORTED = ("mq_version", "mq_last_error", "mq_packed_bytes", "mq_quantize_int8",
            "mq_slice_pack", "mq_linear", "mq_stack_forward", "mq_device_status",
            "mq_release_workspace", "mq_debug_set_wait_limit_ns", "mq_linear_noalloc",
            "mq_quantize_int8_clipped", "mq_linear_container", "mq_ep_overflow_rows",
            "mq_ep_overflow_cols", "mq_linear_ep", "mq_chain_scratch_bytes",
            "mq_chain_forward", "mq_container_save", "mq_container_info", "mq_container_load",
            "mq_chain_scratch_views", "mq_debug_map_table_count")

NOALLOC_SCRATCH_BYTES = 1280 * 1024


class MQError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"mq status {status}: {message}")
        self.status = status


def _check(status: int) -> None:
    if status != MQ_OK:
        raise MQError(status, _last_error().decode(errors="replace"))


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return int(t.data_ptr())


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)


def version() -> int:
    return _version()


def last_error() -> str:
    return _last_error().decode(errors="replace")


def packed_bytes(N: int, K: int, r: int) -> int:
    return int(_packed_bytes(N, K, r))


def quantize_int8(w, dtype: int, N: int, K: int, q, alpha, zero, stream=None) -> None:
    """Eq. 1 per-row MinMax int8 container: q (N x K uint8), alpha, zero (N fp32)."""
    _check(_quantize(_ptr(w), dtype, N, K, _ptr(q), _ptr(alpha), _ptr(zero), _stream(stream)))


def quantize_int8_clipped(w, dtype: int, N: int, K: int, gamma, beta, q, alpha, zero,
                          stream=None) -> None:
    """Eq. 3: OmniQuant-clipped container with per-row gamma, beta (N fp32)."""
    _check(_quantize_clipped(_ptr(w), dtype, N, K, _ptr(gamma), _ptr(beta), _ptr(q), _ptr(alpha),
                             _ptr(zero), _stream(stream)))


def slice_pack(q, N: int, K: int, r: int, packed, stream=None) -> None:
    """Eq. 6 slice of the container at width r, packed as dense r-bit planes."""
    _check(_slice_pack(_ptr(q), N, K, r, _ptr(packed), _stream(stream)))


def linear(x, M: int, K: int, packed, alpha, zero, N: int, r: int, y, stream=None) -> None:
    """y (M x N fp32) = x (M x K bf16) . W_r^T from the packed planes."""
    _check(_linear(_ptr(x), M, K, _ptr(packed), _ptr(alpha), _ptr(zero), N, r, _ptr(y),
                   _stream(stream)))


def linear_container(x, M: int, K: int, q, alpha, zero, N: int, r: int, clamp: bool, y,
                     stream=None) -> None:
    """Slice on load: y = x . W_r^T read straight from the int8 container q,
    sliced by Eq. 6 (clamp=True) or the unclamped Eq. 8 (clamp=False)."""
    _check(_linear_container(_ptr(x), M, K, _ptr(q), _ptr(alpha), _ptr(zero), N, r,
                             1 if clamp else 0, _ptr(y), _stream(stream)))


def ep_overflow_rows(q, N: int, K: int, r: int, row_ptr, stream=None) -> None:
    """Extra Precision list, step 1: row_ptr (N + 1 int32) = scan of the
    per-row counts of positions whose Eq. 8 code exceeds the Eq. 6 code."""
    _check(_ovf_rows(_ptr(q), N, K, r, _ptr(row_ptr), _stream(stream)))


def ep_overflow_cols(q, N: int, K: int, r: int, row_ptr, cols, stream=None) -> None:
    """Extra Precision list, step 2: cols (row_ptr[N] uint16) = those positions."""
    _check(_ovf_cols(_ptr(q), N, K, r, _ptr(row_ptr), _ptr(cols), _stream(stream)))


def linear_ep(x, M: int, K: int, packed, alpha, zero, N: int, r: int, row_ptr, cols, y,
              stream=None) -> None:
    """Eq. 8 (Extra Precision) product: the Eq. 6 planes plus the sparse list."""
    _check(_linear_ep(_ptr(x), M, K, _ptr(packed), _ptr(alpha), _ptr(zero), N, r, _ptr(row_ptr),
                      _ptr(cols), _ptr(y), _stream(stream)))


def chain_scratch_bytes(M: int, D: int, Dkv: int, F: int) -> int:
    return int(_chain_bytes(M, D, Dkv, F))


def chain_scratch_views(M: int, D: int, Dkv: int, F: int) -> dict:
    """Byte offsets of the last layer's intermediates in the chain's scratch."""
    v = ChainViews()
    _check(_chain_views(M, D, Dkv, F, ctypes.byref(v)))
    return {n: int(getattr(v, n)) for n, _ in ChainViews._fields_}


class ChainPlan:
    """Host descriptors of a chained stack, built once and reused. `layers` is
    a list of (r, [qkv, o, gate, up, down]) with each linear a (packed, alpha,
    zero) triple of device tensors."""

    def __init__(self, layers, M: int, D: int, Dkv: int, F: int, head_dim: int):
        self.M, self.D, self.Dkv, self.F, self.hd = M, D, Dkv, F, head_dim
        self.n = len(layers)
        self.arr = (ChainLayer * self.n)()
        for i, (r, lins) in enumerate(layers):
            self.arr[i].r = r
            for j, (p, a, z) in enumerate(lins):
                self.arr[i].packed[j] = _ptr(p)
                self.arr[i].alpha[j] = _ptr(a)
                self.arr[i].zero[j] = _ptr(z)

    def run(self, h, scratch, graph: bool = False, stream=None) -> None:
        """One decode step through every layer: h (M x D fp32) in place."""
        nbytes = scratch.numel() * scratch.element_size()
        _check(_chain(self.arr, self.n, self.M, self.D, self.Dkv, self.F, self.hd, _ptr(h),
                      _ptr(scratch), nbytes, MQ_CHAIN_GRAPH if graph else 0, _stream(stream)))


def save_container(path: str, q, alpha, zero) -> None:
    """Writes the int8 container (q N x K uint8, alpha and zero N fp32; torch
    tensors on any device) to `path` in the library's file format."""
    qh, ah, zh = (t.detach().contiguous().cpu() for t in (q, alpha, zero))
    n, k = qh.shape
    _check(_c_save(os.fsencode(path), qh.data_ptr(), ah.data_ptr(), zh.data_ptr(), n, k))


def container_shape(path: str) -> tuple:
    """(N, K) of a container file."""
    n, k = _i64(0), _i64(0)
    _check(_c_info(os.fsencode(path), ctypes.byref(n), ctypes.byref(k)))
    return n.value, k.value


def load_container(path: str, device=None):
    """Reads a container file into (q, alpha, zero) torch tensors on `device`
    (the host by default); the checksum is verified."""
    import torch
    n, k = container_shape(path)
    q = torch.empty((n, k), dtype=torch.uint8)
    a = torch.empty(n, dtype=torch.float32)
    z = torch.empty(n, dtype=torch.float32)
    _check(_c_load(os.fsencode(path), q.data_ptr(), a.data_ptr(), z.data_ptr(), n, k))
    if device is not None:
        q, a, z = q.to(device), a.to(device), z.to(device)
    return q, a, z


def linear_noalloc(x, M: int, K: int, packed, alpha, zero, N: int, r: int, y, stream=None) -> None:
    """As linear() for 1 <= M <= 32, but working in the library's fixed device
    array instead of allocating a workspace (for callers that cannot allocate).
    Calls that overlap on the GPU share that array and race."""
    _check(_linear_noalloc(_ptr(x), M, K, _ptr(packed), _ptr(alpha), _ptr(zero), N, r, _ptr(y),
                           _stream(stream)))


class StackPlan:
    """The arguments of one Mix'n'Match stack call, marshalled once.

    lins: sequence of (x, packed, alpha, zero, y, N, K); layer_of_lin[i] is
    the layer of linear i and widths[layer] its width. run() then makes the
    same mq_stack_forward call without rebuilding the descriptor arrays.
    The tensors must stay alive (the plan keeps references to them).
    """

    def __init__(self, lins, layer_of_lin, widths, M: int):
        n = len(lins)
        self._keep = list(lins)
        self._arr = (LinearDesc * n)()
        for i, (x, packed, alpha, zero, y, N, K) in enumerate(lins):
            self._arr[i] = LinearDesc(_ptr(x), _ptr(packed), _ptr(alpha), _ptr(zero), _ptr(y), N, K)
        self._lol = (_int * n)(*layer_of_lin)
        self._wd = (_int * len(widths))(*widths)
        self._n, self._nl, self._M = n, len(widths), M

    def run(self, stream=None) -> None:
        _check(_stack(self._arr, self._lol, self._n, self._wd, self._nl, self._M, _stream(stream)))


def stack_forward(lins, layer_of_lin, widths, M: int, stream=None) -> None:
    """Mix'n'Match stack. lins: sequence of (x, packed, alpha, zero, y, N, K)."""
    StackPlan(lins, layer_of_lin, widths, M).run(stream)


def device_status(stream=None) -> None:
    """Synchronizes the stream; raises MQError(MQ_ERR_TIMEOUT) if a kernel gave up a wait."""
    _check(_device_status(_stream(stream)))


def release_workspace() -> None:
    _check(_release())


def debug_set_wait_limit_ns(ns: int) -> None:
    _check(_wait_limit(ns))


def debug_map_table_count() -> int:
    return int(_map_count())


def raw_status(fn_name: str, *args) -> int:
    """Calls a C entry point and returns its status code without raising
    (used by tests of the argument checks)."""
    return {"mq_quantize_int8": _quantize, "mq_slice_pack": _slice_pack,
            "mq_quantize_int8_clipped": _quantize_clipped,
            "mq_linear": _linear, "mq_linear_noalloc": _linear_noalloc,
            "mq_linear_container": _linear_container, "mq_linear_ep": _linear_ep,
            "mq_ep_overflow_rows": _ovf_rows, "mq_ep_overflow_cols": _ovf_cols,
            "mq_container_save": _c_save, "mq_container_load": _c_load}[fn_name](*args)
