"""Many-in-one checkpoints (host side, no GPU): CRC-32C, the documented file
format, loads at every slice count, and rejection of damaged files.

The file format is checked by an independent reader written here from the
format stated in include/mobi.h (struct unpacking, a bitwise CRC-32C), not
through the library's own reader.
"""
import ctypes
import os
import struct

import numpy as np
import pytest

import token_adaptive_mixed_b200 as mobi
from token_adaptive_mixed_b200 import build as mobi_build


@pytest.fixture(scope="module")
def L():
    mobi_build.build()
    return mobi.lib()


def crc32c_bitwise(data: bytes, crc: int = 0) -> int:
    """CRC-32C from its definition: reflected polynomial 0x82F63B78, init and
    final xor 0xFFFFFFFF, one bit at a time."""
    c = crc ^ 0xFFFFFFFF
    for b in data:
        c ^= b
        for _ in range(8):
            c = (c >> 1) ^ 0x82F63B78 if c & 1 else c >> 1
    return c ^ 0xFFFFFFFF


def test_crc32c_check_value(L):
    assert mobi.mobi_crc32c(b"123456789") == 0xE3069283  # the published CRC-32C check value
    assert crc32c_bitwise(b"123456789") == 0xE3069283
    rng = np.random.default_rng(0)
    for n in (1, 7, 8, 9, 63, 64, 1000, 4097):
        data = rng.integers(0, 256, n, dtype=np.uint8).tobytes()
        assert mobi.mobi_crc32c(data) == crc32c_bitwise(data), n
        # continuation: crc(a + b) == crc(b, crc(a))
        assert mobi.mobi_crc32c(data[n // 2:], mobi.mobi_crc32c(data[:n // 2])) == mobi.mobi_crc32c(data)


def packed_arrays(seed, N, K, S, G=128):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 2 ** 32, (S, N, K // 16), dtype=np.uint64).astype(np.uint32).view(np.int32)
    sz = rng.integers(0, 2 ** 32, (S, K // G, N), dtype=np.uint64).astype(np.uint32).view(np.int32)
    return codes, sz


TENSORS = [("layers.0.q", 64, 256, 3), ("layers.0.down", 32, 1152, 2), ("lm_head", 16, 128, 1)]


@pytest.fixture()
def ckpt_file(tmp_path, L):
    arrays = {name: packed_arrays(i, N, K, S) for i, (name, N, K, S) in enumerate(TENSORS)}
    path = tmp_path / "model.mobi"
    mobi.mobi_ckpt_save(path, [(name, *arrays[name]) for name, *_ in TENSORS])
    return path, arrays


def test_format_as_documented(ckpt_file):
    path, arrays = ckpt_file
    raw = path.read_bytes()
    assert raw[:8] == b"MOBICKPT"
    version, count, toff, tbytes, tcrc = struct.unpack_from("<IIQQI", raw, 8)
    assert (version, count, toff, tbytes) == (1, len(TENSORS), 64, 192 * len(TENSORS))
    assert crc32c_bitwise(raw[toff:toff + tbytes]) == tcrc
    for i, (name, N, K, S) in enumerate(TENSORS):
        e = raw[toff + 192 * i: toff + 192 * (i + 1)]
        assert e[:96].split(b"\0")[0].decode() == name
        n, k, g, s, coff, cslice, zoff, zslice = struct.unpack_from("<qqiiQQQQ", e, 96)
        crcs = struct.unpack_from("<8I", e, 96 + 56)
        assert (n, k, g, s) == (N, K, 128, S)
        assert cslice == N * K // 4 and zslice == (K // 128) * N * 4
        assert coff % 4096 == 0 and zoff % 4096 == 0
        codes, sz = arrays[name]
        for sl in range(S):
            cb = raw[coff + sl * cslice: coff + (sl + 1) * cslice]
            zb = raw[zoff + sl * zslice: zoff + (sl + 1) * zslice]
            assert cb == codes[sl].tobytes() and zb == sz[sl].tobytes()
            assert crcs[sl] == crc32c_bitwise(cb) and crcs[4 + sl] == crc32c_bitwise(zb)
        assert all(c == 0 for c in crcs[S:4]) and all(c == 0 for c in crcs[4 + S:])


def test_load_every_slice_count(ckpt_file):
    path, arrays = ckpt_file
    with mobi.MobiCheckpoint(path) as ck:
        assert ck.names() == [t[0] for t in TENSORS]
        assert ck.find("lm_head") == 2 and ck.find("nope") == -1
        expected_read = 0
        for name, N, K, S in TENSORS:
            assert ck.info(ck.find(name)) == (name, N, K, 128, S)
            codes, sz = arrays[name]
            for k in range(1, S + 1):
                c, z = ck.load(name, k)
                assert c.shape == (k, N, K // 16) and z.shape == (k, K // 128, N)
                assert np.array_equal(c.numpy(), codes[:k]) and np.array_equal(z.numpy(), sz[:k])
                expected_read += k * (N * K // 4 + (K // 128) * N * 4)
                assert ck.bytes_read == expected_read  # only the prefix of each block is read
        with pytest.raises(mobi.MobiError, match="INVALID_ARG"):
            ck.load("lm_head", 2)
        with pytest.raises(mobi.MobiError, match="INVALID_ARG"):
            ck.load("layers.0.q", 0)
        with pytest.raises(KeyError):
            ck.load("nope")


def flip_byte(path, offset):
    with open(path, "r+b") as f:
        f.seek(offset)
        b = f.read(1)
        f.seek(offset)
        f.write(bytes([b[0] ^ 0x5A]))


def entry_fields(path, i):
    raw = path.read_bytes()
    return struct.unpack_from("<qqiiQQQQ", raw, 64 + 192 * i + 96)


def test_damaged_slice_is_caught_only_when_read(ckpt_file):
    path, arrays = ckpt_file
    N, K, G, S, coff, cslice, zoff, zslice = entry_fields(path, 0)
    flip_byte(path, coff + cslice + cslice // 2)  # inside slice 2 of the first tensor's codes
    with mobi.MobiCheckpoint(path) as ck:
        c, _ = ck.load(0, 1)  # slice 1 is intact and is all that is read
        assert np.array_equal(c.numpy(), arrays["layers.0.q"][0][:1])
        with pytest.raises(mobi.MobiError, match="IO"):
            ck.load(0, 2)
        assert "checksum" in mobi.mobi_last_error()
        c, _ = ck.load(0, 2, verify=False)  # unchecked: the damaged word comes through
        assert not np.array_equal(c.numpy(), arrays["layers.0.q"][0][:2])


def test_damaged_table_and_foreign_files(ckpt_file, tmp_path):
    path, _ = ckpt_file
    flip_byte(path, 64 + 100)  # inside the first table entry
    with pytest.raises(mobi.MobiError, match="IO"):
        mobi.MobiCheckpoint(path)
    other = tmp_path / "other.bin"
    other.write_bytes(b"not a checkpoint at all" * 10)
    with pytest.raises(mobi.MobiError, match="IO"):
        mobi.MobiCheckpoint(other)
    with pytest.raises(mobi.MobiError, match="IO"):
        mobi.MobiCheckpoint(tmp_path / "missing.mobi")


def rewrite_entry(path, i, fields):
    """Overwrite entry i's size and offset fields and re-seal the table with a
    correct CRC-32C, so only the reader's bounds checks stand between a crafted
    file and out-of-range reads."""
    raw = bytearray(path.read_bytes())
    struct.pack_into("<qqiiQQQQ", raw, 64 + 192 * i + 96, *fields)
    count, toff, tbytes = struct.unpack_from("<IQQ", raw, 12)
    struct.pack_into("<I", raw, 32, crc32c_bitwise(bytes(raw[toff:toff + tbytes])))
    path.write_bytes(bytes(raw))


@pytest.mark.parametrize("case", ["huge_N", "wrapping_codes_offset", "wrapping_sz_offset", "slices_past_end"])
def test_crafted_table_with_valid_crc_is_rejected(ckpt_file, case):
    path, _ = ckpt_file
    N, K, G, S, coff, cslice, zoff, zslice = entry_fields(path, 0)
    if case == "huge_N":  # N * K / 4 no longer fits the bound (and would wrap the slice arithmetic)
        N2 = 1 << 61
        f = (N2, K, G, S, coff, (N2 * K // 4) % (1 << 64), zoff, ((K // G) * N2 * 4) % (1 << 64))
    elif case == "wrapping_codes_offset":  # offset + S * slice wraps past 2^64 to a small number
        f = (N, K, G, S, (1 << 64) - cslice, cslice, zoff, zslice)
    elif case == "wrapping_sz_offset":
        f = (N, K, G, S, coff, cslice, (1 << 64) - zslice, zslice)
    else:  # a valid-looking entry whose last slice runs past the end of the file
        f = (N, K, G, S, path.stat().st_size - cslice, cslice, zoff, zslice)
    rewrite_entry(path, 0, f)
    with pytest.raises(mobi.MobiError, match="IO"):
        mobi.MobiCheckpoint(path)
    assert "corrupt table entry" in mobi.mobi_last_error()


def test_truncated_file(ckpt_file, tmp_path):
    path, _ = ckpt_file
    raw = path.read_bytes()
    short = tmp_path / "short.mobi"
    short.write_bytes(raw[: len(raw) - 4096])
    with pytest.raises(mobi.MobiError, match="IO"):
        mobi.MobiCheckpoint(short)  # the last sz block now runs past the end


def test_save_rejects_bad_tensors(tmp_path, L):
    codes, sz = packed_arrays(0, 16, 128, 2)
    with pytest.raises(mobi.MobiError, match="INVALID_ARG"):
        mobi.mobi_ckpt_save(tmp_path / "a.mobi", [("x", codes, sz), ("x", codes, sz)])  # duplicate name
    with pytest.raises(mobi.MobiError, match="INVALID_ARG"):
        mobi.mobi_ckpt_save(tmp_path / "b.mobi", [("n" * 96, codes, sz)])  # name too long
    assert not os.path.exists(tmp_path / "a.mobi") and not os.path.exists(tmp_path / "b.mobi")
    assert L.mobi_ckpt_save(b"/nonexistent-dir/x.mobi", None, 0, 1, None) == 1
    arr = (mobi.CkptTensor * 1)(mobi.CkptTensor(b"x", ctypes.c_void_p(codes.ctypes.data),
                                                ctypes.c_void_p(sz.ctypes.data), 16, 128, 128, 2))
    assert L.mobi_ckpt_save(b"/nonexistent-dir/x.mobi", arr, 1, 1, None) == 7  # MOBI_ERR_IO


def test_oracle_packed_layer_round_trip(tmp_path, oracle, L):
    """A layer packed by the oracle, stored, and loaded at each precision gives
    the oracle's own slice prefixes back."""
    from token_adaptive_mixed_b200 import workloads as wl
    W = wl.tiny().W
    codes, sz, _ = oracle.pack(W, S=3)
    path = tmp_path / "tiny.mobi"
    mobi.mobi_ckpt_save(path, [("tiny", codes.view(np.int32), sz.view(np.int32))])
    with mobi.MobiCheckpoint(path) as ck:
        for k in (1, 2, 3):
            c, z = ck.load("tiny", k)
            assert np.array_equal(c.numpy().view(np.uint32), codes[:k])
            assert np.array_equal(z.numpy().view(np.uint32), sz[:k])
