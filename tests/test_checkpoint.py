"""Context checkpoint files on the CPU: round trip, the CRC-32 field against the standard
check value and zlib, and the refusals (corruption, truncation, size mismatch, trailing
bytes, bad magic, a failed write leaving nothing behind)."""
import os
import struct
import zlib

import numpy as np
import pytest


@pytest.fixture(scope="module")
def akv():
    from kv_cache_tiering_b200 import build
    build.build()
    from kv_cache_tiering_b200 import akv as mod
    return mod


def _spans(seed=0, sizes=(0, 1, 1000, 65537)):
    rng = np.random.default_rng(seed)
    return [rng.integers(0, 256, size=n, dtype=np.uint8) for n in sizes]


def _read_back(akv, path, sizes):
    out = [np.zeros(n, np.uint8) for n in sizes]
    akv.checkpoint_read(path, [(a, a.nbytes) for a in out])
    return out


def test_round_trip(akv, tmp_path):
    path = str(tmp_path / "ctx.ckpt")
    spans = _spans()
    akv.checkpoint_write(path, [7, 2**63 + 5, 0], [(a, a.nbytes) for a in spans])
    assert not os.path.exists(path + ".tmp")
    meta, sizes = akv.checkpoint_info(path)
    assert meta == [7, 2**63 + 5, 0] and sizes == [a.nbytes for a in spans]
    for a, b in zip(spans, _read_back(akv, path, sizes)):
        assert np.array_equal(a, b)


def test_crc_field_is_crc32(akv, tmp_path):
    path = str(tmp_path / "crc.ckpt")
    data = np.frombuffer(b"123456789", np.uint8).copy()
    akv.checkpoint_write(path, [], [(data, data.nbytes)])
    raw = open(path, "rb").read()
    assert raw[:8] == b"AKVCKPT1"
    version, n_meta, n_spans, zero = struct.unpack_from("<IIII", raw, 8)
    assert (version, n_meta, n_spans, zero) == (1, 0, 1, 0)
    nbytes, crc, zero = struct.unpack_from("<QII", raw, 24)
    assert nbytes == 9 and zero == 0
    assert crc == 0xCBF43926 == zlib.crc32(b"123456789")   # the published CRC-32 check value
    assert raw[40:] == b"123456789"


def _refused(akv, fn):
    with pytest.raises(akv.AkvError) as e:
        fn()
    assert e.value.status == akv.AKV_ERR_INVALID
    return str(e.value)


def test_refusals(akv, tmp_path):
    path = str(tmp_path / "bad.ckpt")
    spans = _spans(1, sizes=(100, 200))
    akv.checkpoint_write(path, [1], [(a, a.nbytes) for a in spans])
    raw = bytearray(open(path, "rb").read())
    sizes = [100, 200]
    # a flipped byte in the second span
    bad = bytearray(raw)
    bad[-5] ^= 0x40
    open(path, "wb").write(bad)
    assert "CRC-32" in _refused(akv, lambda: _read_back(akv, path, sizes))
    # truncated
    open(path, "wb").write(raw[:-10])
    assert "truncated" in _refused(akv, lambda: _read_back(akv, path, sizes))
    # trailing bytes
    open(path, "wb").write(raw + b"x")
    assert "trailing" in _refused(akv, lambda: _read_back(akv, path, sizes))
    # the caller's buffer sizes differ from the recorded ones
    open(path, "wb").write(raw)
    assert "size" in _refused(akv, lambda: _read_back(akv, path, [100, 201]))
    assert "count" in _refused(akv, lambda: _read_back(akv, path, [100]))
    # not a checkpoint
    bad = bytearray(raw)
    bad[0:8] = b"NOTACKPT"
    open(path, "wb").write(bad)
    assert "magic" in _refused(akv, lambda: akv.checkpoint_info(path))
    # the intact file still reads
    open(path, "wb").write(raw)
    for a, b in zip(spans, _read_back(akv, path, sizes)):
        assert np.array_equal(a, b)


def test_failed_write_leaves_nothing(akv, tmp_path):
    path = str(tmp_path / "no_such_dir" / "x.ckpt")
    data = np.zeros(16, np.uint8)
    _refused(akv, lambda: akv.checkpoint_write(path, [], [(data, 16)]))
    assert not os.path.exists(path) and not os.path.exists(path + ".tmp")
