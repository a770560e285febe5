"""Host half of the C-ABI library against the oracle (no GPU needed).

The library's codebook must reach the optimal cost the oracle computes; the
oracle re-encodes the block from the library's code lengths and must get the
library's stream, gaps, chunk positions and sign|mantissa bytes byte for byte;
every 16-bit window walked through the library's two-level tables must give
the oracle's first code.  Page: "DFloat11: lossless BFloat16 compression".
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import workloads
import huffman_decode_b200 as df11
from huffman_decode_b200 import df11 as binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "df11.h")).read()
    return sorted(set(re.findall(r"^(?:df11_status|const char \*|uint64_t|uint32_t)\s*(df11_\w+)\s*\(", src, re.M)))


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert set(names) == set(df11.EXPORTED_SYMBOLS)
    df11.load_library()                       # builds it if needed
    lib = ctypes.CDLL(df11.library_path())    # a fresh handle, no prototypes set
    for n in names:
        assert hasattr(lib, n), n
    lib.df11_status_string.restype = ctypes.c_char_p
    assert lib.df11_status_string(0) == b"ok"


def _flat(mats):
    return np.concatenate([np.ascontiguousarray(m, dtype=np.uint16).reshape(-1) for m in mats])


def check_format_parity(mats, bytes_per_thread=8, cap=16):
    """Library artifact == the oracle's artifact built from the library's
    code lengths; the library's lengths reach the oracle's optimal cost."""
    threads_per_chunk = 32
    cb = df11.build_codebook(mats, cap)
    hb = df11.compress(cb, mats, threads_per_chunk, bytes_per_thread)
    assert df11.validate(hb) == 0
    w = _flat(mats)
    e, s = oracle.split(w)
    counts = oracle.histogram(e)
    assert np.array_equal(cb.counts(), counts)
    L = cb.lengths()
    best = oracle.code_lengths(counts, cap)
    assert oracle.total_bits(counts, L) == oracle.total_bits(counts, best)
    assert int(L.max()) <= cap
    ob = oracle.compress_block(mats, cap=cap, threads_per_chunk=threads_per_chunk,
                               bytes_per_thread=bytes_per_thread, lengths=L)
    assert np.array_equal(cb.codes(), ob.codes)
    h = hb.header
    assert (h.total_bits, h.n_elements, h.n_chunks) == (ob.total_bits, w.size, ob.n_chunks)
    assert np.array_equal(hb.exp_stream, ob.stream)
    gaps = np.empty(hb.gaps.size * 2, np.uint8)
    gaps[0::2], gaps[1::2] = hb.gaps & 15, hb.gaps >> 4
    assert np.array_equal(gaps, ob.gap)
    assert np.array_equal(hb.counts, ob.thread_count)
    assert np.array_equal(hb.chunk_pos, ob.pos)
    assert np.array_equal(hb.signmant[: w.size], ob.signmant)
    assert not hb.signmant[w.size:].any()
    check_tables(hb.lut, int(h.n_tables), L)
    return cb, hb, ob


def check_tables(lut, n_tables, lengths):
    """Walk every 16-bit window through the two-level tables as the format
    defines them and compare with the oracle's bit-by-bit first code."""
    sym, ln = oracle.first_code_table(lengths)
    t = lut.reshape(-1, 256)[:n_tables].astype(np.int64)
    v = np.arange(65536)
    e = t[0][v >> 8]
    ptr = (e & 0x8000) != 0
    assert np.all((e[ptr] & 0xFF) >= 1) and np.all((e[ptr] & 0xFF) < n_tables)
    e[ptr] = t[e[ptr] & 0xFF, v[ptr] & 0xFF]
    assert not np.any(e & 0x8000)                     # no third level
    nocode = (e & 0x4000) != 0
    assert np.array_equal(nocode, ln == 0)
    ok = ~nocode
    assert np.array_equal(e[ok] & 0xFF, sym[ok])
    assert np.array_equal((e[ok] >> 8) & 0x1F, ln[ok])


SMALL_WORKLOADS = {
    "single_1024x1024": lambda: workloads.single_matrix(0),
    "llama_block_div64": lambda: workloads.llama_block(1000, scale_div=64),
    "flux_block_div64": lambda: workloads.flux_block(5000, scale_div=64),
    "heavy_tail_512": lambda: workloads.heavy_tail(4001, (512, 512)),
    "single_exponent_512": lambda: workloads.single_exponent(4002, (512, 512)),
    "uniform_bits_512": lambda: workloads.uniform_bits(4003, (512, 512)),
    "many_tables_1m": lambda: workloads.many_tables(4004, 1 << 20),
}


@pytest.mark.parametrize("name", sorted(SMALL_WORKLOADS))
@pytest.mark.parametrize("bpt", [8, 16])
def test_format_parity_small_workloads(name, bpt):
    mats = [m for _, m in SMALL_WORKLOADS[name]()]
    check_format_parity(mats, bytes_per_thread=bpt)


@pytest.mark.parametrize("cap", [8, 9, 12, 15, 16])
def test_codebook_optimal_under_cap(cap):
    """Fibonacci-like counts push the natural Huffman depth to 23; the
    library's lengths must meet the oracle's package-merge optimum."""
    fib = [1, 1]
    while len(fib) < 24:
        fib.append(fib[-1] + fib[-2])
    rng = np.random.default_rng(cap)
    e = np.repeat(np.arange(100, 124, dtype=np.uint16), fib)
    rng.shuffle(e)
    w = (e << np.uint16(7)) | rng.integers(0, 256, e.size).astype(np.uint16) & np.uint16(0x807F)
    check_format_parity([w], cap=cap)


@pytest.mark.parametrize("seed", range(6))
def test_codebook_random_alphabets(seed):
    rng = np.random.default_rng(50 + seed)
    n_sym = int(rng.integers(2, 257))
    syms = rng.choice(256, n_sym, replace=False).astype(np.uint16)
    p = rng.dirichlet(np.full(n_sym, float(rng.uniform(0.05, 2.0))))
    e = rng.choice(syms, 20000, p=p)
    w = (e << np.uint16(7)) | (rng.integers(0, 65536, e.size).astype(np.uint16) & np.uint16(0x807F))
    check_format_parity([w], cap=int(rng.integers(8, 17)) if n_sym <= 256 else 16)


def test_all_bf16_patterns_and_tiny_sizes():
    allw = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    check_format_parity([allw])
    for n in (1, 2, 7, 8, 9, 15, 16, 17):
        for bpt in (8, 16):
            check_format_parity([allw[12345: 12345 + n]], bytes_per_thread=bpt)
    # several matrices, including a one-element one, in caller order
    check_format_parity([allw[:5], allw[40000:40001], allw[100:1100]])


@pytest.mark.parametrize("delta", [-1, 0, 1])
@pytest.mark.parametrize("bpt", [8, 16])
def test_chunk_boundary(delta, bpt):
    """Stream lengths one bit under, at and over a whole chunk (32 slices)."""
    chunk_bits = 32 * 8 * bpt
    # two symbols of 1 bit each: total bits == element count
    n = chunk_bits + delta
    rng = np.random.default_rng(7)
    e = np.where(rng.random(n) < 0.5, 0x7A, 0x7B).astype(np.uint16)
    w = (e << np.uint16(7)) | rng.integers(0, 128, n).astype(np.uint16)
    cb, hb, ob = check_format_parity([w], bytes_per_thread=bpt)
    assert hb.header.total_bits == n
    assert hb.header.n_chunks == (1 if delta <= 0 else 2)


def test_decode_of_library_artifact_by_oracle():
    mats = [m for _, m in workloads.heavy_tail(4001, (256, 512))]
    cb = df11.build_codebook(mats)
    hb = df11.compress(cb, mats)
    out = oracle.decode_block(hb.exp_stream, hb.n_elements, cb.lengths(), hb.signmant)
    assert np.array_equal(out, _flat(mats))


# ----------------------------------------------------------- error paths

def test_build_codebook_errors():
    w = np.arange(100, dtype=np.uint16)
    for cap in (0, 7, 17, 32):
        with pytest.raises(df11.DF11Error) as ei:
            df11.build_codebook([w], cap)
        assert ei.value.status == 1
    with pytest.raises(df11.DF11Error) as ei:
        df11.build_codebook([np.zeros(0, np.uint16)])
    assert ei.value.status == 1
    lib = df11.load_library()
    cb = binding.Codebook()
    assert lib.df11_build_codebook(None, None, 0, 16, ctypes.byref(cb)) == 1


def test_compress_errors():
    rng = np.random.default_rng(3)
    w = rng.integers(0, 65536, 5000).astype(np.uint16)
    cb = df11.build_codebook([w])
    with pytest.raises(df11.DF11Error) as ei:               # different data
        df11.compress(cb, [w[::-1].copy() ^ np.uint16(0x0080)])
    assert ei.value.status == 1
    for tpc in (0, 16, 64, 128, 256, 300):
        with pytest.raises(df11.DF11Error):
            df11.compress(cb, [w], threads_per_chunk=tpc)
    for bpt in (0, 4, 12, 32):
        with pytest.raises(df11.DF11Error):
            df11.compress(cb, [w], bytes_per_thread=bpt)
    # a buffer one entry short
    hb = df11.compress(cb, [w])
    blk = hb.c_struct()
    blk.chunk_pos_count -= 1
    lib = df11.load_library()
    arrs, ptrs, numel = binding._mats_args([w])
    ly = binding.Layout(32, 8)
    assert lib.df11_compress(ctypes.byref(cb), ctypes.byref(ly), ptrs, numel, 1,
                             ctypes.byref(blk)) == 2


def _fresh_block():
    mats = [m for _, m in workloads.llama_block(1002, scale_div=256)]
    cb = df11.build_codebook(mats)
    return df11.compress(cb, mats)


def test_validate_flags_corruption():
    hb = _fresh_block()
    assert df11.validate(hb) == 0
    bad = _fresh_block(); bad.chunk_pos[1], bad.chunk_pos[2] = bad.chunk_pos[2], bad.chunk_pos[1]
    assert df11.validate(bad) == 4
    bad = _fresh_block(); bad.chunk_pos[-1] -= 1
    assert df11.validate(bad) == 4
    bad = _fresh_block()                       # a gap past the end of the stream
    g = bad.gaps.size * 2 - 1
    assert 8 * bad.header.bytes_per_thread * g >= bad.header.total_bits
    bad.gaps[g // 2] |= 0x50
    assert df11.validate(bad) == 4
    bad = _fresh_block(); bad.gaps[0] |= 0x01  # thread 0 always starts at bit 0
    assert df11.validate(bad) == 4
    bad = _fresh_block(); bad.lut[5] = 0x8000 | 200
    assert df11.validate(bad) == 4
    bad = _fresh_block(); bad.lut[0] = 0
    assert df11.validate(bad) == 4
    bad = _fresh_block(); bad.header.n_chunks += 1
    assert df11.validate(bad) == 4
    bad = _fresh_block(); bad.header.total_bits = bad.header.n_elements - 1
    assert df11.validate(bad) == 4
    # the header claims a shortest code longer than one the tables hold
    bad = _fresh_block()
    assert bad.header.min_code_len == 2
    bad.header.min_code_len = 3
    assert df11.validate(bad) == 4
    bad = _fresh_block(); bad.header.min_code_len = 0
    assert df11.validate(bad) == 4


def test_header_min_code_len_matches_codebook():
    for mats in ([m for _, m in workloads.llama_block(1002, scale_div=256)],
                 [m for _, m in workloads.single_exponent(4002, (64, 64))],
                 [m for _, m in workloads.uniform_bits(4003, (64, 64))]):
        cb = df11.build_codebook(mats)
        hb = df11.compress(cb, mats)
        L = cb.lengths()
        assert hb.header.min_code_len == int(L[L > 0].min())


def test_decompress_rejects_bad_arguments_before_any_cuda_call():
    """Host-side checks only; every case fails before the library touches the
    CUDA runtime, so this runs without a GPU."""
    hb = _fresh_block()
    lib = df11.load_library()
    fake = 1 << 20                                   # 16-byte aligned, never dereferenced

    def dev_block(**over):
        b = binding._Block()
        b.hdr = hb.header
        for name in ("exp_stream", "gaps", "chunk_pos", "signmant", "lut"):
            setattr(b, name, fake)
        b.exp_stream_bytes = hb.exp_stream.nbytes
        b.gaps_bytes = hb.gaps.nbytes
        b.chunk_pos_count = hb.chunk_pos.size
        b.signmant_bytes = hb.signmant.nbytes
        b.lut_entries = hb.lut.size
        for k, v in over.items():
            setattr(b, k, v)
        return b

    n = hb.n_elements
    call = lambda b, out=fake, cap=n, err=None: lib.df11_decompress_async(
        ctypes.byref(b), out, cap, err, None)
    assert lib.df11_decompress_async(None, fake, n, None, None) == 1
    assert call(dev_block(), out=None) == 1
    assert call(dev_block(), cap=n - 1) == 1                       # too little room
    assert call(dev_block(exp_stream=None)) == 1
    assert call(dev_block(gaps_bytes=hb.gaps.nbytes - 1)) == 1
    assert call(dev_block(chunk_pos_count=hb.chunk_pos.size - 1)) == 1
    assert call(dev_block(lut_entries=hb.lut.size - 1)) == 1
    assert call(dev_block(exp_stream=fake + 4)) == 1               # misaligned
    assert call(dev_block(gaps=fake + 8)) == 1
    assert call(dev_block(signmant=fake + 8)) == 1
    assert call(dev_block(), out=fake + 2) == 1
    assert call(dev_block(), err=fake + 1) == 1
    h = binding.Header.from_buffer_copy(hb.header)
    h.threads_per_chunk = 64
    assert call(dev_block(hdr=h)) == 1
    h = binding.Header.from_buffer_copy(hb.header)
    h.bytes_per_thread = 4
    assert call(dev_block(hdr=h)) == 1
    h = binding.Header.from_buffer_copy(hb.header)
    h.n_chunks += 1
    assert call(dev_block(hdr=h)) == 1
    h = binding.Header.from_buffer_copy(hb.header)
    h.n_tables = 0
    assert call(dev_block(hdr=h)) == 1
    for bad_min in (0, 17):
        h = binding.Header.from_buffer_copy(hb.header)
        h.min_code_len = bad_min
        assert call(dev_block(hdr=h)) == 1
    # the CTA-capped entry point runs the same checks
    capped = lambda b, cap=n: lib.df11_decompress_async_ctas(ctypes.byref(b), fake, cap, None, 8, None)
    assert lib.df11_decompress_async_ctas(None, fake, n, None, 8, None) == 1
    assert capped(dev_block(), cap=n - 1) == 1
    assert capped(dev_block(signmant=fake + 8)) == 1
    # and so does the entry point with a scheduling workspace, which must
    # also be 16-byte aligned
    with_ws = lambda b, ws, cap=n: lib.df11_decompress_async_ws(ctypes.byref(b), fake, cap, None, 0, ws, None)
    assert lib.df11_decompress_async_ws(None, fake, n, None, 0, fake, None) == 1
    assert with_ws(dev_block(), fake + 4) == 1
    assert with_ws(dev_block(), fake, cap=n - 1) == 1
    assert with_ws(dev_block(exp_stream=fake + 8), fake) == 1
    # the chunk-range entry point: the same checks, and a non-empty range
    # inside the block, all before any CUDA call
    nch = int(hb.header.n_chunks)
    rng = lambda b, c0, c1, ws=None: lib.df11_decompress_range_async(ctypes.byref(b), c0, c1, fake, n, None,
                                                                     ws, None)
    assert lib.df11_decompress_range_async(None, 0, 1, fake, n, None, None, None) == 1
    assert rng(dev_block(), 0, 0) == 1
    assert rng(dev_block(), 3, 2) == 1
    assert rng(dev_block(), 0, nch + 1) == 1
    assert rng(dev_block(), nch, nch + 1) == 1
    assert rng(dev_block(), 0, 1, ws=fake + 8) == 1
    assert rng(dev_block(exp_stream=fake + 8), 0, 1) == 1
    # the bounded-wait self-test checks its arguments before launching
    assert lib.df11_selftest_bounded_wait(0, fake, None) == 1
    assert lib.df11_selftest_bounded_wait(4097, fake, None) == 1
    assert lib.df11_selftest_bounded_wait(16, None, None) == 1
    assert lib.df11_selftest_bounded_wait(16, fake + 2, None) == 1


def test_pipeline_rejects_bad_arguments_before_any_cuda_call():
    """df11_pipeline_*: argument checks that need no CUDA runtime."""
    lib = df11.load_library()
    h = ctypes.c_void_p()
    assert lib.df11_pipeline_create(0, ctypes.byref(h)) == 1
    assert lib.df11_pipeline_create(65, ctypes.byref(h)) == 1
    assert lib.df11_pipeline_create(2, None) == 1
    assert lib.df11_pipeline_destroy(None) == 1
    fake = 1 << 20
    b = binding._Block()
    assert lib.df11_pipeline_upload(None, 0, ctypes.byref(b), ctypes.byref(b), None) == 1
    assert lib.df11_pipeline_decode(None, 0, ctypes.byref(b), fake, 16, None, 0, None, None) == 1
    assert lib.df11_pipeline_acquire(None, 0, None) == 1
    assert lib.df11_pipeline_release(None, 0, None) == 1


# ------------------------------------------- codebook from a histogram

@pytest.mark.parametrize("name", ["single_1024x1024", "heavy_tail_512", "uniform_bits_512",
                                  "single_exponent_512"])
def test_codebook_from_histogram_equals_data_pass(name):
    """The histogram entry point (used with the GPU histogram) builds exactly
    the codebook the data pass builds."""
    mats = [m for _, m in SMALL_WORKLOADS[name]()]
    a = df11.build_codebook(mats)
    counts = oracle.histogram(oracle.split(_flat(mats))[0])
    b = df11.build_codebook_from_histogram(counts)
    assert bytes(a) == bytes(b)


def test_codebook_from_histogram_errors():
    with pytest.raises(df11.DF11Error):
        df11.build_codebook_from_histogram(np.zeros(256, np.uint64))
    h = np.zeros(256, np.uint64); h[3] = 5
    with pytest.raises(df11.DF11Error):
        df11.build_codebook_from_histogram(h, 7)
    h[4] = 1 << 32
    with pytest.raises(df11.DF11Error) as ei:
        df11.build_codebook_from_histogram(h)
    assert ei.value.status == 3


def test_compress_device_rejects_bad_arguments_before_any_cuda_call():
    mats = [m for _, m in workloads.llama_block(1002, scale_div=256)]
    cb = df11.build_codebook(mats)
    lib = df11.load_library()
    n = int(cb.n_elements)
    ly = binding.Layout(32, 16)
    z = df11.compress_sizes(cb)
    fake = 1 << 20
    b = binding._Block()
    for name in binding.ARRAYS:
        setattr(b, name, fake)
    b.exp_stream_bytes, b.gaps_bytes, b.counts_bytes = z.exp_stream_bytes, z.gaps_bytes, z.counts_bytes
    b.chunk_pos_count, b.signmant_bytes, b.lut_entries = z.chunk_pos_count, z.signmant_bytes, z.lut_entries
    scratch = df11.compress_device_scratch_bytes(n)
    assert scratch >= 12 * ((n + 8191) // 8192)
    call = lambda **kw: lib.df11_compress_device(
        ctypes.byref(cb), ctypes.byref(kw.get("ly", ly)), kw.get("inp", fake), kw.get("n", n),
        ctypes.byref(kw.get("blk", b)), kw.get("scr", fake), kw.get("scrn", scratch),
        kw.get("err", None), None)
    assert call(inp=None) == 1
    assert call(n=n + 1) == 1
    assert call(scr=None) == 1
    assert call(scrn=scratch - 1) == 2
    assert call(inp=fake + 2) == 1
    assert call(err=fake + 2) == 1
    assert call(ly=binding.Layout(32, 4)) == 1
    short = binding._Block.from_buffer_copy(b)
    short.gaps_bytes -= 1
    assert call(blk=short) == 2
    short = binding._Block.from_buffer_copy(b)
    short.counts_bytes -= 1
    assert call(blk=short) == 2
    nocounts = binding._Block.from_buffer_copy(b)
    nocounts.counts = None
    assert call(blk=nocounts) == 1
    assert lib.df11_histogram_device(None, n, fake, None) == 1
    assert lib.df11_histogram_device(fake, 0, fake, None) == 1
    assert lib.df11_histogram_device(fake + 2, n, fake, None) == 1


# ------------------------------------------------------------- checksums
# "DFloat11: lossless BFloat16 compression", "How to run it in production":
# checksum every artifact.  The library's CRC-32C list must equal the
# oracle's bit-by-bit CRC of every 4096-byte segment of every array.

def _oracle_list(hb):
    return oracle.block_checksums(hb.exp_stream, hb.gaps, hb.counts, hb.chunk_pos, hb.signmant, hb.lut)


@pytest.mark.parametrize("name", ["single_1024x1024", "heavy_tail_512", "single_exponent_512"])
def test_checksum_list_equals_oracle(name):
    mats = [m for _, m in SMALL_WORKLOADS[name]()]
    cb = df11.build_codebook(mats)
    hb = df11.compress(cb, mats)
    got = df11.checksum(hb)
    ref = _oracle_list(hb)
    assert df11.checksum_count(hb) == ref.size
    assert np.array_equal(got, ref)


def _oracle_chunk_sums(hb):
    h = hb.header
    return oracle.chunk_sums(hb.exp_stream, hb.gaps, hb.counts, hb.chunk_pos, hb.signmant, hb.lut,
                             h.n_tables, h.bytes_per_thread, h.n_chunks)


@pytest.mark.parametrize("name", ["single_1024x1024", "heavy_tail_512", "single_exponent_512", "tiny"])
@pytest.mark.parametrize("bpt", [8, 16])
def test_chunk_sums_equal_oracle(name, bpt):
    """df11_chunk_sums (the library's word-level code) against the oracle's
    bit-by-bit definition, every chunk, both slice widths."""
    mats = ([workloads.single_matrix(3, shape=(3, 5))[0][1]] if name == "tiny"
            else [m for _, m in SMALL_WORKLOADS[name]()])
    cb = df11.build_codebook(mats)
    hb = df11.compress(cb, mats, 32, bpt)
    got = df11.chunk_sums(hb)
    assert got.size == hb.header.n_chunks
    assert np.array_equal(got, _oracle_chunk_sums(hb))


def test_chunk_sums_reject_bad_arguments():
    hb = _fresh_block()
    lib = df11.load_library()
    b = hb.c_struct()
    n = int(hb.header.n_chunks)
    out = np.empty(n + 1, np.uint32)
    assert lib.df11_chunk_sums(ctypes.byref(b), out.ctypes.data, n) == 0
    assert lib.df11_chunk_sums(ctypes.byref(b), out.ctypes.data, n + 1) == 1
    assert lib.df11_chunk_sums(ctypes.byref(b), None, n) == 1
    assert lib.df11_chunk_sums(None, out.ctypes.data, n) == 1
    pos = hb.chunk_pos.copy()
    pos[1], pos[2] = pos[2], pos[1] - 1        # decreasing positions
    bad = df11.HostBlock(header=hb.header, exp_stream=hb.exp_stream, gaps=hb.gaps, counts=hb.counts,
                         chunk_pos=pos, signmant=hb.signmant, lut=hb.lut)
    bb = bad.c_struct()
    assert lib.df11_chunk_sums(ctypes.byref(bb), out.ctypes.data, n) == 1
    # the verified decode's host-side checks, before any CUDA call
    fake = 1 << 20
    d = binding._Block()
    d.hdr = hb.header
    for name in ("exp_stream", "gaps", "counts", "chunk_pos", "signmant", "lut"):
        setattr(d, name, fake)
    d.exp_stream_bytes, d.gaps_bytes, d.counts_bytes = hb.exp_stream.nbytes, hb.gaps.nbytes, hb.counts.nbytes
    d.chunk_pos_count, d.signmant_bytes, d.lut_entries = hb.chunk_pos.size, hb.signmant.nbytes, hb.lut.size
    m = hb.n_elements
    v = lib.df11_decompress_verified_async
    assert v(ctypes.byref(d), fake, m, fake, None, None, None, None) == 1          # no sums
    assert v(ctypes.byref(d), fake, m, None, fake, None, None, None) == 1          # no error word
    assert v(ctypes.byref(d), fake, m, fake, fake + 2, None, None, None) == 1      # misaligned sums
    assert v(ctypes.byref(d), fake, m, fake, fake, fake + 4, None, None) == 1      # misaligned first_bad
    assert v(ctypes.byref(d), None, m, fake, fake, None, None, None) == 1
    assert v(None, fake, m, fake, fake, None, None, None) == 1
    assert v(ctypes.byref(d), fake, m - 1, fake, fake, None, None, None) == 1      # too little room


def test_crc32c_equals_oracle_any_length_and_offset():
    rng = np.random.default_rng(11)
    buf = rng.integers(0, 256, 20000, dtype=np.uint8)
    for start in (0, 1, 3, 7, 8, 13):
        for n in (0, 1, 2, 7, 8, 9, 15, 16, 17, 4095, 4096, 4097, 12345):
            d = buf[start:start + n]
            assert df11.crc32c(d) == oracle.crc32c(d), (start, n)


def test_checksum_rejects_bad_arguments():
    hb = _fresh_block()
    lib = df11.load_library()
    b = hb.c_struct()
    n = df11.checksum_count(hb)
    out = np.empty(n + 1, np.uint32)
    assert lib.df11_checksum(ctypes.byref(b), out.ctypes.data, n + 1) == 1
    assert lib.df11_checksum(ctypes.byref(b), None, n) == 1
    assert lib.df11_checksum(None, out.ctypes.data, n) == 1
    assert lib.df11_checksum_count(None) == 0
    fake = 1 << 20
    d = binding._Block()
    d.hdr = hb.header
    for name in ("exp_stream", "gaps", "chunk_pos", "signmant", "lut"):
        setattr(d, name, fake)
    d.exp_stream_bytes, d.gaps_bytes = hb.exp_stream.nbytes, hb.gaps.nbytes
    d.chunk_pos_count, d.signmant_bytes, d.lut_entries = hb.chunk_pos.size, hb.signmant.nbytes, hb.lut.size
    # host-side checks of the GPU calls, before any CUDA call
    assert lib.df11_checksum_device_async(ctypes.byref(d), fake, n + 1, None) == 1
    assert lib.df11_checksum_device_async(ctypes.byref(d), None, n, None) == 1
    assert lib.df11_verify_device_async(ctypes.byref(d), fake, n, None, None, None) == 1
    assert lib.df11_verify_device_async(ctypes.byref(d), fake, n, fake, fake + 4, None) == 1
    d.signmant = fake + 8
    assert lib.df11_checksum_device_async(ctypes.byref(d), fake, n, None) == 1


def test_decode_gemv_rejects_bad_arguments_before_any_cuda_call():
    """df11_decode_gemv_async: matrix table and token checks need no GPU."""
    hb = _fresh_block()
    lib = df11.load_library()
    fake = 1 << 20
    d = binding._Block()
    d.hdr = hb.header
    for name in ("exp_stream", "gaps", "chunk_pos", "signmant", "lut"):
        setattr(d, name, fake)
    d.exp_stream_bytes, d.gaps_bytes = hb.exp_stream.nbytes, hb.gaps.nbytes
    d.chunk_pos_count, d.signmant_bytes, d.lut_entries = hb.chunk_pos.size, hb.signmant.nbytes, hb.lut.size
    shapes = [m.shape for _, m in workloads.llama_block(1002, scale_div=256)]

    def table(shp, x=fake, y=fake):
        arr = (binding.GemvMatrix * len(shp))()
        for i, (r, c) in enumerate(shp):
            arr[i] = binding.GemvMatrix(r, c, x, y)
        return arr

    call = lambda arr, n, t, ws=None: lib.df11_decode_gemv_async(ctypes.byref(d), arr, n, t, None, ws, None)
    good = table(shapes)
    assert sum(r * c for r, c in shapes) == hb.n_elements
    assert call(good, len(shapes), 0) == 1                      # no tokens
    assert call(good, len(shapes), 9) == 1                      # more than 8
    assert call(good, 0, 1) == 1
    assert call(good, len(shapes) - 1, 1) == 1                  # does not cover the block
    assert call(table(shapes, x=fake + 8), len(shapes), 1) == 1 # misaligned activations
    assert call(table(shapes, y=fake + 2), len(shapes), 1) == 1
    bad = list(shapes)
    bad[0] = (bad[0][0] * 2, bad[0][1] // 2 + 4)                # cols not a multiple of 8
    assert call(table(bad), len(bad), 1) == 1
    assert lib.df11_decode_gemv_async(None, good, len(shapes), 1, None, None, None) == 1
    assert call(good, len(shapes), 1, ws=fake + 8) == 1         # misaligned workspace


# ------------------------------------------------ decoder's multi-code table

def _oracle_multi_entry(k, sym, ln, window_bits=11):
    """The entry for window k (first stream bit = bit 0 of k) from the
    oracle's first-code table: the whole codes the window starts with, at
    most four, as rotated exponents and their total length | 8 x count << 16."""
    m = 0
    for b in range(window_bits):
        m |= ((k >> b) & 1) << (window_bits - 1 - b)        # MSB-first window
    used = n = syms = 0
    while n < 4:
        v = ((m << used) << (16 - window_bits)) & 0xFFFF     # unknown bits read as 0
        s, l = int(sym[v]), int(ln[v])
        if s < 0 or used + l > window_bits:
            break
        syms |= (((s >> 1) | ((s & 1) << 7)) & 0xFF) << (8 * n)
        n += 1
        used += l
    y = used | (8 * n << 16) if n else 0x80000000
    return syms | (y << 32)


@pytest.mark.parametrize("name", ["single_1024x1024", "heavy_tail_1024", "uniform_bits_1024",
                                  "single_exponent_1024", "many_tables"])
def test_decode_table_equals_oracle_walk(name):
    """df11_build_decode_table: every one of the 2048 entries equals a walk
    of the window with the oracle's canonical first-code table (the codes
    the window starts with and their lengths), for codebooks with short and
    long codes, many sub-tables and a single symbol ("Architecture":
    hierarchical lookup tables; "How it works": canonical codes)."""
    mats = {
        "single_1024x1024": lambda: workloads.single_matrix(0),
        "heavy_tail_1024": lambda: workloads.heavy_tail(4001, (1024, 1024)),
        "uniform_bits_1024": lambda: workloads.uniform_bits(4003, (1024, 1024)),
        "single_exponent_1024": lambda: workloads.single_exponent(4002, (1024, 1024)),
        "many_tables": lambda: workloads.many_tables(),
    }[name]()
    mats = [m for _, m in mats]
    cb = df11.build_codebook(mats)
    hb = df11.compress(cb, mats)
    tab = df11.build_decode_table(hb.lut, hb.header.n_tables, hb.header.min_code_len)
    sym, ln = oracle.first_code_table(cb.lengths())
    want = np.array([_oracle_multi_entry(k, sym, ln) for k in range(2048)], np.uint64)
    bad = np.nonzero(tab != want)[0]
    assert bad.size == 0, f"{bad.size} entries differ, first {bad[:4]}: {tab[bad[:4]]} vs {want[bad[:4]]}"


def test_decode_table_reads_malformed_tables_as_no_code():
    """Entries the decoder sanitises (a pointer inside a sub-table, a
    pointer to a missing table, a leaf shorter than the shortest code) end
    the walk exactly where a "no code" entry would; bad arguments are
    refused."""
    mats = [m for _, m in workloads.heavy_tail(4001, (1024, 1024))]
    cb = df11.build_codebook(mats)
    hb = df11.compress(cb, mats)
    nt, ml = hb.header.n_tables, hb.header.min_code_len
    good = df11.build_decode_table(hb.lut, nt, ml)
    lut = hb.lut.copy()
    root = int(np.nonzero(lut[:256] & 0x8000)[0][0])          # a root pointer
    lut[root] = 0x8000 | nt                                   # to a table that does not exist
    bad = df11.build_decode_table(lut, nt, ml)
    # windows whose first 8 bits are that prefix now start with no code
    for k in range(2048):
        first8 = int(''.join(str((k >> b) & 1) for b in range(8)), 2)
        if first8 == root:
            assert bad[k] == np.uint64(0x80000000 << 32)
    assert np.any(bad != good)
    with pytest.raises(df11.DF11Error):
        df11.build_decode_table(hb.lut, 0, ml)
    with pytest.raises(df11.DF11Error):
        df11.build_decode_table(hb.lut, nt, 0)
    with pytest.raises(df11.DF11Error):
        df11.build_decode_table(hb.lut, nt, 17)


def test_preferred_bytes_per_thread_rule():
    """8-byte slices for a 1-bit shortest code or a block with fewer 16-byte
    chunks than the decoder's resident warps; 16 otherwise (the rule
    include/df11.h states)."""
    one_bit = [m for _, m in workloads.single_exponent(4002, (256, 256))]
    assert df11.preferred_bytes_per_thread(df11.build_codebook(one_bit), 148) == 8
    small = [m for _, m in workloads.single_matrix(0)]
    cb = df11.build_codebook(small)
    assert min(l for l in cb.lengths() if l) >= 2
    chunks16 = -(-int(cb.total_bits) // (32 * 128))
    assert chunks16 < 148 * 46
    assert df11.preferred_bytes_per_thread(cb, 148) == 8
    # the same codebook on a GPU with few SMs: enough chunks for every warp
    sm_few = chunks16 // 46
    assert df11.preferred_bytes_per_thread(cb, sm_few) == 16
    assert df11.preferred_bytes_per_thread(cb, sm_few + 1) == 8
    lib = df11.load_library()
    assert lib.df11_preferred_bytes_per_thread(None, 148) == 0
    assert lib.df11_preferred_bytes_per_thread(ctypes.byref(cb), 0) == 0
