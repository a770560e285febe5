"""CPU oracle for the DFloat11 exponent codec -- TEST INFRASTRUCTURE ONLY.

A plain, slow, single-threaded restatement of the method on the page
"DFloat11: lossless BFloat16 compression" (sections "What it is",
"Architecture" and "How it works: the core algorithm"; the artifact checksum
of "How to run it in production").  The arithmetic lives
in ``df11_oracle.c`` (plain C, compiled here with gcc); this module only
marshals numpy arrays.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import it.  It shares no code with the
``huffman_decode_b200`` library and neither imports the other.

Functions with a pin in ``tests/test_oracle_pins.py``: every one below.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "df11_oracle.c")
_HDR = os.path.join(_HERE, "df11_oracle.h")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libdf11_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle's C source into a shared library (gcc, -O2)."""
    newest_src = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= newest_src:
        return _LIB_PATH
    os.makedirs(_BUILD_DIR, exist_ok=True)
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(
        ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-shared", "-fPIC",
         "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    U64 = ctypes.c_uint64
    U32 = ctypes.c_uint32
    I = ctypes.c_int
    sig = {
        "orc_split": (None, [P, U64, P, P]),
        "orc_join": (None, [P, P, U64, P]),
        "orc_histogram_add": (None, [P, U64, P]),
        "orc_entropy": (ctypes.c_double, [P]),
        "orc_huffman_lengths": (I, [P, P]),
        "orc_package_merge_lengths": (I, [P, I, P]),
        "orc_code_lengths": (I, [P, I, P]),
        "orc_canonical_codes": (I, [P, P]),
        "orc_total_bits": (U64, [P, P]),
        "orc_encode": (I, [P, U64, P, P, P, U64, P]),
        "orc_decode": (I, [P, U64, U64, U64, P, P, P]),
        "orc_first_code_table": (I, [P, P, P]),
        "orc_metadata": (I, [P, U64, P, U32, U32, U64, P, P, P]),
        "orc_chunk_sums": (I, [P, P, P, P, P, U64, P, U32, U32, U64, P]),
        "orc_crc32c": (U32, [P, U64]),
        "orc_segment_crcs": (U64, [P, U64, U64, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _u8(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.uint8)


# ------------------------------------------------------------------ fields

def split(w: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """BF16 bit patterns -> (exponent bytes, sign|mantissa bytes)."""
    w = np.ascontiguousarray(w, dtype=np.uint16).reshape(-1)
    e = np.empty(w.size, np.uint8)
    s = np.empty(w.size, np.uint8)
    _load().orc_split(_ptr(w), w.size, _ptr(e), _ptr(s))
    return e, s


def join(e: np.ndarray, s: np.ndarray) -> np.ndarray:
    e = _u8(e).reshape(-1)
    s = _u8(s).reshape(-1)
    assert e.size == s.size
    w = np.empty(e.size, np.uint16)
    _load().orc_join(_ptr(e), _ptr(s), e.size, _ptr(w))
    return w


# -------------------------------------------------------------- statistics

def histogram(exps) -> np.ndarray:
    """256-bin exponent counts summed over one array or a list of arrays."""
    if isinstance(exps, np.ndarray):
        exps = [exps]
    counts = np.zeros(256, np.uint64)
    for e in exps:
        e = _u8(e).reshape(-1)
        _load().orc_histogram_add(_ptr(e), e.size, _ptr(counts))
    return counts


def entropy(counts: np.ndarray) -> float:
    counts = np.ascontiguousarray(counts, dtype=np.uint64)
    return float(_load().orc_entropy(_ptr(counts)))


def huffman_lengths(counts: np.ndarray) -> np.ndarray:
    counts = np.ascontiguousarray(counts, dtype=np.uint64)
    ln = np.zeros(256, np.uint8)
    if _load().orc_huffman_lengths(_ptr(counts), _ptr(ln)) < 0:
        raise ValueError("no live symbol")
    return ln


def package_merge_lengths(counts: np.ndarray, cap: int) -> np.ndarray:
    counts = np.ascontiguousarray(counts, dtype=np.uint64)
    ln = np.zeros(256, np.uint8)
    if _load().orc_package_merge_lengths(_ptr(counts), cap, _ptr(ln)) < 0:
        raise ValueError("package-merge needs 2 <= symbols <= 2^cap")
    return ln


def code_lengths(counts: np.ndarray, cap: int = 16) -> np.ndarray:
    counts = np.ascontiguousarray(counts, dtype=np.uint64)
    ln = np.zeros(256, np.uint8)
    if _load().orc_code_lengths(_ptr(counts), cap, _ptr(ln)) < 0:
        raise ValueError("cannot build code lengths")
    return ln


def canonical_codes(lengths: np.ndarray) -> np.ndarray:
    lengths = _u8(lengths)
    codes = np.zeros(256, np.uint32)
    if _load().orc_canonical_codes(_ptr(lengths), _ptr(codes)) != 0:
        raise ValueError("lengths violate Kraft's inequality")
    return codes


def total_bits(counts: np.ndarray, lengths: np.ndarray) -> int:
    counts = np.ascontiguousarray(counts, dtype=np.uint64)
    return int(_load().orc_total_bits(_ptr(counts), _ptr(_u8(lengths))))


# --------------------------------------------------------------- bitstream

def encode(exp: np.ndarray, lengths: np.ndarray, codes: np.ndarray,
           stream_bytes: int | None = None) -> tuple[np.ndarray, int]:
    """MSB-first bitstream of the exponents; returns (bytes, bit count)."""
    exp = _u8(exp).reshape(-1)
    lengths = _u8(lengths)
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    if stream_bytes is None:
        stream_bytes = (int(lengths[exp].astype(np.uint64).sum()) + 7) // 8 if exp.size else 0
    stream = np.zeros(max(stream_bytes, 1), np.uint8)
    tb = ctypes.c_uint64(0)
    rc = _load().orc_encode(_ptr(exp), exp.size, _ptr(lengths), _ptr(codes),
                            _ptr(stream), stream_bytes, ctypes.addressof(tb))
    if rc != 0:
        raise ValueError("encode failed")
    return stream[:stream_bytes], int(tb.value)


def decode(stream: np.ndarray, n: int, lengths: np.ndarray,
           start_bit: int = 0) -> tuple[np.ndarray, int]:
    """Bit-by-bit canonical decode of n symbols; returns (exponents, end bit)."""
    stream = _u8(stream).reshape(-1)
    out = np.empty(max(n, 1), np.uint8)
    end = ctypes.c_uint64(0)
    rc = _load().orc_decode(_ptr(stream) if stream.size else 0, stream.size, start_bit, n,
                            _ptr(_u8(lengths)), _ptr(out), ctypes.addressof(end))
    if rc != 0:
        raise ValueError("stream does not decode")
    return out[:n], int(end.value)


def first_code_table(lengths: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """For each 16-bit window: (first symbol or -1, its code length or 0)."""
    sym = np.empty(65536, np.int16)
    ln = np.empty(65536, np.uint8)
    if _load().orc_first_code_table(_ptr(_u8(lengths)), _ptr(sym), _ptr(ln)) != 0:
        raise ValueError("bad lengths")
    return sym, ln


def metadata(exp: np.ndarray, lengths: np.ndarray, threads_per_chunk: int,
             bytes_per_thread: int, n_chunks: int) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(per-thread gap, per-thread code count, both unpacked; per-chunk output
    positions incl. the end)."""
    exp = _u8(exp).reshape(-1)
    gap = np.zeros(n_chunks * threads_per_chunk, np.uint8)
    count = np.zeros(n_chunks * threads_per_chunk, np.uint8)
    pos = np.zeros(n_chunks + 1, np.uint32)
    rc = _load().orc_metadata(_ptr(exp) if exp.size else 0, exp.size, _ptr(_u8(lengths)),
                              threads_per_chunk, bytes_per_thread, n_chunks,
                              _ptr(gap), _ptr(count), _ptr(pos))
    if rc != 0:
        raise ValueError("metadata failed")
    return gap, count, pos


# ----------------------------------------------------- whole-block helpers

@dataclass
class OracleBlock:
    """The oracle's own DF11 artifact for one block of matrices."""
    lengths: np.ndarray      # uint8[256]
    codes: np.ndarray        # uint32[256]
    counts: np.ndarray       # uint64[256]
    total_bits: int
    n_elements: int
    n_chunks: int
    stream: np.ndarray       # uint8, zero padded to n_chunks*T*W + pad bytes
    gap: np.ndarray          # uint8 per thread (unpacked)
    thread_count: np.ndarray  # uint8 per thread: codes starting in its slice
    pos: np.ndarray          # uint32[n_chunks + 1]
    signmant: np.ndarray     # uint8[n_elements]


def compress_block(mats, cap: int = 16, threads_per_chunk: int = 32,
                   bytes_per_thread: int = 8, pad_bytes: int = 16,
                   lengths: np.ndarray | None = None) -> OracleBlock:
    """Split, histogram over all matrices, code lengths under `cap` (or the
    given lengths), canonical codes, bitstream and metadata, in the page's order.
    The stream holds n_chunks*T*W bytes plus `pad_bytes` zero bytes."""
    w = np.concatenate([np.ascontiguousarray(m, dtype=np.uint16).reshape(-1) for m in mats])
    e, s = split(w)
    counts = histogram(e)
    if lengths is None:
        lengths = code_lengths(counts, cap)
    codes = canonical_codes(lengths)
    tb = total_bits(counts, lengths)
    chunk_bits = threads_per_chunk * bytes_per_thread * 8
    n_chunks = (tb + chunk_bits - 1) // chunk_bits
    stream_bytes = n_chunks * threads_per_chunk * bytes_per_thread + pad_bytes
    stream, tb2 = encode(e, lengths, codes, stream_bytes)
    assert tb2 == tb
    gap, thread_count, pos = metadata(e, lengths, threads_per_chunk, bytes_per_thread, n_chunks)
    return OracleBlock(lengths=lengths, codes=codes, counts=counts, total_bits=tb,
                       n_elements=w.size, n_chunks=n_chunks, stream=stream, gap=gap,
                       thread_count=thread_count, pos=pos, signmant=s)


def decode_block(stream: np.ndarray, n_elements: int, lengths: np.ndarray,
                 signmant: np.ndarray) -> np.ndarray:
    """Serial bit-by-bit decode of a whole block, joined back into BF16."""
    e, _ = decode(stream, n_elements, lengths)
    return join(e, _u8(signmant)[:n_elements])


# ------------------------------------------------------------- checksum

CRC_SEGMENT = 4096


def crc32c(data) -> int:
    """CRC-32C of the raw bytes of `data` (bytes or numpy array), bit by bit."""
    a = _u8(np.frombuffer(bytes(data), np.uint8) if isinstance(data, (bytes, bytearray))
            else np.ascontiguousarray(data).view(np.uint8).reshape(-1))
    return int(_load().orc_crc32c(_ptr(a) if a.size else None, a.size))


def segment_crcs(data, seg: int = CRC_SEGMENT) -> np.ndarray:
    """CRC-32C of every `seg`-byte segment of the raw bytes of `data`."""
    a = _u8(np.ascontiguousarray(data).view(np.uint8).reshape(-1))
    out = np.empty(max(1, (a.size + seg - 1) // seg), np.uint32)
    k = _load().orc_segment_crcs(_ptr(a) if a.size else None, a.size, seg, _ptr(out))
    return out[:k]


def block_checksums(exp_stream, gaps, counts, chunk_pos, signmant, lut, seg: int = CRC_SEGMENT) -> np.ndarray:
    """The checksum list of a block: segment CRCs of its six arrays in the
    order exp_stream, gaps, counts, chunk_pos, signmant, lut (raw
    little-endian bytes of each array as given)."""
    return np.concatenate([segment_crcs(a, seg) for a in (exp_stream, gaps, counts, chunk_pos, signmant, lut)])


# ----------------------------------------------------------- chunk sums

def chunk_sums(stream, gaps, counts, chunk_pos, signmant, lut, n_tables: int, bytes_per_thread: int,
               n_chunks: int) -> np.ndarray:
    """The per-chunk sums of a block (see orc_chunk_sums in df11_oracle.h):
    gaps packed two per byte, counts one byte per thread, chunk_pos uint32."""
    stream, gaps, counts, signmant = _u8(stream), _u8(gaps), _u8(counts), _u8(signmant)
    pos = np.ascontiguousarray(chunk_pos, dtype=np.uint32)
    lut = np.ascontiguousarray(lut, dtype=np.uint16)
    out = np.zeros(max(int(n_chunks), 1), np.uint32)
    if pos.size < int(n_chunks) + 1 or stream.size < 32 * int(bytes_per_thread) * int(n_chunks) or \
            gaps.size < 16 * int(n_chunks) or counts.size < 32 * int(n_chunks) or lut.size < 256 * int(n_tables):
        raise ValueError("chunk_sums: arrays shorter than the block")
    rc = _load().orc_chunk_sums(_ptr(stream), _ptr(gaps), _ptr(counts), _ptr(pos), _ptr(signmant), signmant.size,
                                _ptr(lut), int(n_tables), int(bytes_per_thread), int(n_chunks), _ptr(out))
    if rc != 0:
        raise ValueError("chunk_sums failed")
    return out[: int(n_chunks)]
