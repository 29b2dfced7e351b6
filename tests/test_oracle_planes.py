"""Pins for the dense r-bit plane layout.

* hand-computed words for hand-made rows (tests/golden/plane_words.txt),
  written from the layout's index formula, not produced by the oracle;
* the vectorized packer equals the Python-integer packer bit for bit;
* unpack(pack(codes)) is the identity for random and edge codes;
* the size is N*K*r/8 bytes (dense), and r = 8 stores the container bytes.
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
WIDTHS = [8, 6, 4, 3, 2]


def _cases():
    out, cur = [], None
    with open(os.path.join(GOLDEN, "plane_words.txt")) as f:
        for ln in f:
            if not ln.strip() or ln.startswith("#"):
                continue
            tag, *vals = ln.split()
            if tag == "case":
                cur = {"r": int(vals[0])}
                out.append(cur)
            elif tag == "codes":
                cur["codes"] = [int(v) for v in vals]
            elif tag == "words":
                cur["words"] = [int(v, 16) for v in vals]
    return out


def test_golden_words():
    cases = _cases()
    assert {c["r"] for c in cases} == set(WIDTHS)
    for c in cases:
        want = np.array(c["words"], dtype="<u4").view(np.uint8)
        got = oracle.pack_rows(np.array([c["codes"]]), c["r"])
        assert np.array_equal(got, want), c["r"]
        assert oracle.pack_rows_bigint([c["codes"]], c["r"]) == want.tobytes()


@pytest.mark.parametrize("r", WIDTHS)
def test_vectorized_equals_bigint(r):
    codes = np.random.default_rng(r).integers(0, 1 << r, size=(5, 96))
    assert oracle.pack_rows(codes, r).tobytes() == oracle.pack_rows_bigint(codes, r)


@pytest.mark.parametrize("r", WIDTHS)
def test_round_trip(r):
    rng = np.random.default_rng(10 + r)
    for codes in [rng.integers(0, 1 << r, size=(9, 128)),
                  np.zeros((3, 32), np.int64),
                  np.full((3, 64), (1 << r) - 1),
                  np.tile(np.arange(32) % (1 << r), (2, 2))]:
        n, k = codes.shape
        packed = oracle.pack_rows(codes, r)
        assert packed.size == oracle.packed_bytes(n, k, r) == n * k * r // 8
        assert np.array_equal(oracle.unpack_rows(packed, n, k, r), codes)


def test_full_width_is_container_bytes():
    q = np.random.default_rng(1).integers(0, 256, size=(4, 64))
    assert np.array_equal(oracle.pack_rows(q, 8), q.astype(np.uint8).reshape(-1))


def test_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle.pack_rows(np.zeros((1, 48), np.int64), 4)
    with pytest.raises(ValueError):
        oracle.pack_rows(np.full((1, 32), 4), 2)
    with pytest.raises(ValueError):
        oracle.plane_widths(5)
