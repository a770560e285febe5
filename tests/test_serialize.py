"""A block as one flat buffer (df11_serialize / df11_deserialize), CPU only.

The container holds the block header, the six arrays and the CRC-32C of
every 4096-byte segment of them ("DFloat11: lossless BFloat16 compression",
"How to run it in production": checksum artifacts on download and after
every copy).  Checks: a round trip gives back every array byte for byte and
the oracle decodes the loaded block to the input bits; any flipped bit in
the header, the arrays or the checksum list, a truncated or padded buffer, a
wrong magic or version is refused (DF11_ERR_CORRUPT) and a flip inside an
array names its segment.
"""
import numpy as np
import pytest

import oracle
import workloads
import huffman_decode_b200 as df11
from huffman_decode_b200 import df11 as binding

ARRAYS = binding.ARRAYS
BLOCKS = {
    "llama_div256": lambda: workloads.llama_block(1003, scale_div=256),
    "heavy_tail_256": lambda: workloads.heavy_tail(4001, (256, 256)),
    "single_exponent_64": lambda: workloads.single_exponent(4002, (64, 64)),
    "tiny_3x8": lambda: workloads.single_matrix(5, shape=(3, 8)),
}


def _block(name, bpt=16):
    mats = [m for _, m in BLOCKS[name]()]
    cb = df11.build_codebook(mats)
    return mats, cb, df11.compress(cb, mats, 32, bpt)


@pytest.mark.parametrize("name", sorted(BLOCKS))
@pytest.mark.parametrize("bpt", [8, 16])
def test_round_trip_is_exact_and_decodes(name, bpt, tmp_path):
    mats, cb, hb = _block(name, bpt)
    data = hb.to_bytes()
    assert len(data) % 4 == 0 and data[:8] == b"DF11BLK\0"
    path = tmp_path / "block.df11"
    hb.save(path)
    got = df11.HostBlock.load(path)
    assert bytes(got.header) == bytes(hb.header)
    for a in ARRAYS:
        assert np.array_equal(getattr(got, a).view(np.uint8), getattr(hb, a).view(np.uint8)), a
    ref = oracle.decode_block(got.exp_stream, got.n_elements, cb.lengths(), got.signmant)
    assert np.array_equal(ref, np.concatenate([m.reshape(-1) for m in mats]))
    assert got.to_bytes() == data


def _array_ranges(hb, data):
    """Byte range of every array inside the buffer (16-byte aligned, in order)."""
    at, out = 128, {}
    for a in ARRAYS:
        n = getattr(hb, a).nbytes
        out[a] = (at, at + n)
        at = (at + n + 15) & ~15
    return out, at


def _refused(buf):
    with pytest.raises(df11.DF11Error) as e:
        df11.HostBlock.from_bytes(bytes(buf))
    assert e.value.status == binding.DF11_ERR_CORRUPT
    return e.value


def test_every_region_is_covered():
    _, _, hb = _block("llama_div256")
    data = hb.to_bytes()
    ranges, crc_off = _array_ranges(hb, data)
    rng = np.random.default_rng(11)
    # the header: every byte, its zero padding included
    for i in range(0, 128):
        buf = bytearray(data)
        buf[i] ^= 1 << int(rng.integers(0, 8))
        _refused(buf)
    # the arrays: ends and random bytes; the error names the segment
    first_seg = {}
    k = 0
    for a in ARRAYS:
        first_seg[a] = k
        k += (getattr(hb, a).nbytes + 4095) // 4096
    for a, (lo, hi) in ranges.items():
        for off in sorted({lo, hi - 1, int(rng.integers(lo, hi))}):
            buf = bytearray(data)
            buf[off] ^= 1 << int(rng.integers(0, 8))
            e = _refused(buf)
            assert e.first_bad_segment == first_seg[a] + (off - lo) // 4096, (a, off)
    # the zero padding after each array
    for a, (lo, hi) in ranges.items():
        nxt = (hi + 15) & ~15
        if nxt > hi:
            buf = bytearray(data)
            buf[hi] ^= 1
            _refused(buf)
    # the checksum list itself
    for off in (crc_off, len(data) - 1):
        buf = bytearray(data)
        buf[off] ^= 0x80
        _refused(buf)


def test_truncated_padded_or_foreign_buffers_are_refused():
    _, _, hb = _block("heavy_tail_256")
    data = hb.to_bytes()
    for cut in (0, 7, 127, 128, len(data) // 2, len(data) - 1):
        _refused(data[:cut])
    _refused(data + b"\0" * 4)
    buf = bytearray(data)
    buf[8] = 1                  # another version (the header CRC no longer matches)
    _refused(buf)
    _refused(b"NOTDF11!" + data[8:])


def test_null_arguments():
    lib = df11.load_library()
    import ctypes
    blk = binding._Block()
    assert lib.df11_deserialize(None, 0, ctypes.byref(blk), None) == binding.DF11_ERR_INVALID_ARGUMENT
    assert lib.df11_serialize(None, None, 0) == binding.DF11_ERR_INVALID_ARGUMENT
    assert lib.df11_serialized_bytes(None) == 0
    _, _, hb = _block("tiny_3x8")
    b = hb.c_struct()
    n = lib.df11_serialized_bytes(ctypes.byref(b))
    buf = (ctypes.c_uint8 * n)()
    assert lib.df11_serialize(ctypes.byref(b), buf, n - 1) == binding.DF11_ERR_BUFFER_TOO_SMALL
    assert lib.df11_serialize(ctypes.byref(b), buf, n) == 0
