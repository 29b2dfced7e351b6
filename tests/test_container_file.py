"""The int8 container file (mq_container_save / info / load): host-side I/O,
so these run on the CPU. A round trip is bit-exact; a corrupt, truncated,
padded or foreign file is refused with MQ_ERR_IO; a file of another shape
with MQ_ERR_INVALID_ARG."""
import os
import zlib

import numpy as np
import pytest
import torch

import nested_bit_weight_int8_b200 as mq
import oracle
import synth


def _container(n=37, k=96, seed=0):
    w = synth.f32_from_bf16_bits(synth.gaussian_weights(n, k, seed)).astype(np.float64)
    q, a, z = oracle.quantize_minmax(w)
    return torch.from_numpy(q), torch.from_numpy(a), torch.from_numpy(z)


def test_round_trip_bit_exact(tmp_path):
    q, a, z = _container()
    p = str(tmp_path / "c.mqc")
    mq.save_container(p, q, a, z)
    assert mq.container_shape(p) == (37, 96)
    q2, a2, z2 = mq.load_container(p)
    assert torch.equal(q, q2)
    assert np.array_equal(a.numpy().view(np.uint32), a2.numpy().view(np.uint32))
    assert np.array_equal(z.numpy().view(np.uint32), z2.numpy().view(np.uint32))


def test_layout_and_checksum_are_as_documented(tmp_path):
    # the header, the three arrays in order, and a standard CRC-32 of all of it
    q, a, z = _container(5, 32, 1)
    p = str(tmp_path / "c.mqc")
    mq.save_container(p, q, a, z)
    raw = open(p, "rb").read()
    body = (b"MQC8" + np.uint32(1).tobytes() + np.int64(5).tobytes() + np.int64(32).tobytes()
            + q.numpy().tobytes() + a.numpy().tobytes() + z.numpy().tobytes())
    assert raw[:-4] == body
    assert int.from_bytes(raw[-4:], "little") == zlib.crc32(body)


@pytest.mark.parametrize("damage", ["flip", "truncate", "append", "magic"])
def test_damaged_files_are_refused(tmp_path, damage):
    q, a, z = _container(9, 64, 2)
    p = str(tmp_path / "c.mqc")
    mq.save_container(p, q, a, z)
    raw = bytearray(open(p, "rb").read())
    if damage == "flip":
        raw[24 + 100] ^= 0x10
    elif damage == "truncate":
        raw = raw[:-7]
    elif damage == "append":
        raw += b"\0"
    else:
        raw[0:4] = b"XXXX"
    open(p, "wb").write(bytes(raw))
    with pytest.raises(mq.MQError) as e:
        mq.load_container(p)
    assert e.value.status == mq.MQ_ERR_IO


def test_shape_mismatch_and_bad_arguments(tmp_path):
    q, a, z = _container(9, 64, 3)
    p = str(tmp_path / "c.mqc")
    mq.save_container(p, q, a, z)
    qq = torch.empty((9, 32), dtype=torch.uint8)
    st = mq.raw_status("mq_container_load", os.fsencode(p), qq.data_ptr(), a.data_ptr(), z.data_ptr(), 9, 32)
    assert st == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_container_save", os.fsencode(p), None, a.data_ptr(), z.data_ptr(), 9, 64) \
        == mq.MQ_ERR_INVALID_ARG
    assert mq.raw_status("mq_container_save", os.fsencode(p), q.data_ptr(), a.data_ptr(), z.data_ptr(), 0, 64) \
        == mq.MQ_ERR_INVALID_ARG
    st = mq.raw_status("mq_container_save", os.fsencode(str(tmp_path / "no" / "dir" / "c.mqc")),
                       q.data_ptr(), a.data_ptr(), z.data_ptr(), 9, 64)
    assert st == mq.MQ_ERR_IO
    with pytest.raises(mq.MQError) as e:
        mq.container_shape(str(tmp_path / "missing.mqc"))
    assert e.value.status == mq.MQ_ERR_IO


def test_save_replaces_atomically_and_leaves_no_temporary(tmp_path):
    """A save writes path.tmp.<pid>, closes it and renames it over path: an
    existing file is replaced whole, and no temporary stays behind."""
    q, a, z = _container(11, 64, 4)
    p = str(tmp_path / "c.mqc")
    mq.save_container(p, q, a, z)
    q2, a2, z2 = _container(11, 64, 5)
    mq.save_container(p, q2, a2, z2)
    assert sorted(os.listdir(tmp_path)) == ["c.mqc"]
    q3, _, _ = mq.load_container(p)
    assert torch.equal(q3, q2)


def test_failed_save_leaves_the_target_untouched(tmp_path):
    """When the rename cannot happen (the target is a non-empty directory),
    the save fails with MQ_ERR_IO, the target is as it was and the temporary
    file is removed."""
    q, a, z = _container(7, 32, 6)
    target = tmp_path / "c.mqc"
    target.mkdir()
    (target / "keep").write_bytes(b"x")
    with pytest.raises(mq.MQError) as e:
        mq.save_container(str(target), q, a, z)
    assert e.value.status == mq.MQ_ERR_IO
    assert sorted(os.listdir(tmp_path)) == ["c.mqc"]
    assert (target / "keep").read_bytes() == b"x"
