"""Dense r-bit planes: the storage layout of a sliced width.

The pages fix only that a slice of width r is stored as r-bit integers
("Mix'n'Match and Interpolative Slicing"; "int2/int3 require custom
kernels", section 5.4) and that one int8 container serves every width. The
byte layout is this library's own, chosen so that a GPU register can hold two
neighbouring codes in its two 16-bit halves. It is dense: N*K*r/8 bytes.

A width r is split into planes of power-of-two bit widths b:
  r = 8 -> (8)        r = 4 -> (4)        r = 2 -> (2)
  r = 3 -> (2, 1)     r = 6 -> (4, 2)
Plane 0 holds the low b0 bits of every code, plane 1 (if any) the code
shifted right by b0. Planes are stored one after the other; each plane is
row-major with a row pitch of K*b/8 bytes.

Within a plane, row n is a run of little-endian 32-bit words; word i carries
codes j = i*C .. i*C + C - 1, C = 32 / b. Local code u = j - i*C sits at
  b = 8:        bits [8u, 8u + 8)                       (plain bytes)
  b in {1,2,4}: bits [16*(u % 2) + b*(u // 2), ... + b)  (even codes in the low
                half-word, odd codes in the high half-word)
So r = 8 stores the container bytes unchanged (S(q, 8) = q).
"""
from __future__ import annotations

import numpy as np

_PLANES = {8: (8,), 4: (4,), 2: (2,), 3: (2, 1), 6: (4, 2)}


def plane_widths(r: int) -> tuple:
    if r not in _PLANES:
        raise ValueError("r must be one of 8, 6, 4, 3, 2")
    return _PLANES[r]


def bit_position(u: int, b: int) -> int:
    """Bit offset of local code u inside its 32-bit word, plane width b."""
    if b == 8:
        return 8 * u
    return 16 * (u % 2) + b * (u // 2)


def packed_bytes(n: int, k: int, r: int) -> int:
    if k % 32:
        raise ValueError("K must be a multiple of 32")
    return n * k * r // 8


def _plane_codes(codes: np.ndarray, r: int):
    """Split codes into the per-plane fields (low bits first)."""
    widths = plane_widths(r)
    out, shift = [], 0
    for b in widths:
        out.append((codes >> shift) & ((1 << b) - 1))
        shift += b
    return list(zip(widths, out))


def pack_rows_bigint(codes, r: int) -> bytes:
    """Reference packer with Python integers (small inputs): builds every word
    by placing each code at its bit position, then emits little-endian bytes."""
    codes = [[int(v) for v in row] for row in codes]
    n = len(codes)
    k = len(codes[0]) if n else 0
    if k % 32:
        raise ValueError("K must be a multiple of 32")
    out = bytearray()
    shift = 0
    for b in plane_widths(r):
        per_word = 32 // b
        for row in codes:
            for i in range(k // per_word):
                word = 0
                for u in range(per_word):
                    field = (row[i * per_word + u] >> shift) & ((1 << b) - 1)
                    word |= field << bit_position(u, b)
                out += word.to_bytes(4, "little")
        shift += b
    return bytes(out)


def pack_rows(codes: np.ndarray, r: int) -> np.ndarray:
    """Vectorized packer (same index function as pack_rows_bigint).

    codes: N x K integers in [0, 2^r). Returns a uint8 array of N*K*r/8 bytes.
    """
    codes = np.asarray(codes, dtype=np.int64)
    n, k = codes.shape
    if k % 32:
        raise ValueError("K must be a multiple of 32")
    if codes.size and (codes.min() < 0 or codes.max() >= (1 << r)):
        raise ValueError("codes out of range for r")
    parts = []
    for b, field in _plane_codes(codes, r):
        per_word = 32 // b
        f = field.reshape(n, k // per_word, per_word).astype(np.uint64)
        words = np.zeros((n, k // per_word), dtype=np.uint64)
        for u in range(per_word):
            words |= f[:, :, u] << np.uint64(bit_position(u, b))
        parts.append(words.astype("<u4").reshape(-1).view(np.uint8))
    return np.concatenate(parts) if parts else np.zeros(0, np.uint8)


def unpack_rows(packed: np.ndarray, n: int, k: int, r: int) -> np.ndarray:
    """Inverse of pack_rows: returns the N x K codes."""
    packed = np.ascontiguousarray(np.asarray(packed, dtype=np.uint8))
    if packed.size != packed_bytes(n, k, r):
        raise ValueError("packed size does not match N*K*r/8")
    codes = np.zeros((n, k), dtype=np.int64)
    offset, shift = 0, 0
    for b in plane_widths(r):
        per_word = 32 // b
        nbytes = n * k * b // 8
        words = packed[offset:offset + nbytes].view("<u4").astype(np.int64)
        words = words.reshape(n, k // per_word)
        field = np.zeros((n, k // per_word, per_word), dtype=np.int64)
        for u in range(per_word):
            field[:, :, u] = (words >> bit_position(u, b)) & ((1 << b) - 1)
        codes |= field.reshape(n, k) << shift
        offset += nbytes
        shift += b
    return codes
